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
#define DSA_ERR_NO_DEVICE -7      /* no current CUDA device, or it is not sm_100 */
#define DSA_ERR_LAUNCH -8         /* the CUDA runtime rejected a launch or a copy */
#define DSA_ERR_CONFIG -9         /* kernel attribute set-up failed on this device */

#define DSA_TOPK_MAX_K 2048

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
 *              affect the result). A row may be read up to 12 bytes past its
 *              last valid element, never crossing that element's 16-byte
 *              aligned block.
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
 * Ownership: the caller owns every buffer; the library allocates no device
 * memory per call and keeps no pointer after returning. Buffers must stay
 * valid until the stream reaches the call. The call can be captured in a CUDA
 * graph once the device has seen one uncaptured call (that first call sets
 * per-device kernel attributes).
 *
 * Errors: argument errors return before any launch; DSA_ERR_LAUNCH carries a
 * CUDA runtime failure of the launch. A device-side wait that exceeds its
 * time limit records a flag readable with dsa_topk_device_status().
 */
int dsa_topk(const float* logits, int64_t row_stride, const int32_t* lengths,
             int64_t num_rows, int32_t k, int32_t* out_idx, dsa_stream_t stream);

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
 * that share one row (1 = one CTA per row, persistent over rows); grid = CTAs
 * launched. Either output pointer may be NULL. Returns DSA_OK or an error
 * code as dsa_topk would.
 */
int dsa_topk_plan(int64_t num_rows, int64_t row_stride, int32_t k,
                  int32_t* cluster_size, int32_t* grid);

/*
 * dsa_topk_device_status -- sticky device-side status bits of the current
 * device (bit 0: a pipeline wait timed out). Synchronises the device. With
 * clear != 0 the bits are reset to 0 afterwards. Returns DSA_OK or
 * DSA_ERR_LAUNCH.
 */
int dsa_topk_device_status(uint32_t* status, int clear);

/* Human-readable text for a return code (static storage). */
const char* dsa_topk_strerror(int code);

/* Library version as an integer: major*10000 + minor*100 + patch. */
int dsa_topk_version(void);

#ifdef __cplusplus
}
#endif

#endif /* DSA_TOPK_H_ */
