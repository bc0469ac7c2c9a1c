/*
 * mxscale.h -- C ABI of libmxscale: MXFP8 E8M0 scale factors -> per-group
 * 128x4 blocked ("swizzled") layout, on NVIDIA B200 (sm_100a).
 *
 * The operation (pytorch/ao pull requests on MXFP8 MoE training):
 *   - "[mxfp8 moe training] compute prefix sum of group sizes inside kernel
 *     intead of precomputing" (#3285), Context and Changes: the padded start
 *     of every group is a prefix sum of padded group sizes, computed inside
 *     the kernel, with no host precompute and no device-to-host copy.
 *   - "[mxfp8 moe training] fallback cuda kernel for when input doesn't meet 2d
 *     TMA constraints" (#3708), Context: groups along M; a pipelined TMA kernel
 *     when the row stride is a multiple of 16 bytes, a simpler kernel for any
 *     other width (e.g. 44 columns), chosen per input.
 *   - "[mxfp8 moe training] add bench script for scale conversion to blocked
 *     format kernels for groups along K" (#3604): groups along K, each group
 *     made of 128x4 scale-factor tiles.
 *   - "Add CuTeDSL MXFP8 K-groups scale rearrange kernel" (#4704), review,
 *     "Additional findings": padding is zero; empty groups add nothing; the
 *     grid is over-provisioned by one chunk per group.
 *
 * Layout.  Scales are uint8 (E8M0), row-major (rows x cols) with a row
 * stride in bytes; one scale per 32 data elements.  A group's padded matrix
 * is cut into 128x4 tiles of 512 bytes, ordered row-block-major then
 * column-block-minor; element (r, c) of a tile sits at byte
 * (r%32)*16 + (r/32)*4 + c.
 *   - Groups along M (forward / dgrad): group g is rows [E'[g-1], E'[g]),
 *     padded to a multiple of 128 rows and roundup(cols, 4) columns; group g's
 *     blocked rows start at row P_g = sum_{h<g} roundup(n_h, 128) of one
 *     matrix roundup(cols, 4) wide.
 *   - Groups along K (wgrad): group g is columns [E'[g-1], E'[g]), padded to
 *     W_g = roundup(w_g, 4) columns and R = roundup(rows, 128) rows; group g's
 *     blocked matrix (R x W_g) is stored contiguously at byte R * sum_{h<g} W_h.
 *   Group ends E are int32 in device memory, cumulative (end of group g), in
 *   rows (M) or scale columns (K).  They are read only on the device and are
 *   clamped there, never rejected: E'[-1] = 0, E'[g] = min(max(E[g], E'[g-1]), T)
 *   with T = rows (M) or cols (K).  Rows (M) or columns (K) past E'[G-1] are
 *   ignored.  Every byte of the output allocation is written: real bytes,
 *   zero padding, and a zero tail after the last group; the caller need not
 *   clear `out`.
 *
 * Ownership and streams.  The caller owns every buffer.  The library never
 * allocates, frees or synchronises, never reads device memory on the host,
 * and launches only on `stream`, so every call may be captured in a CUDA
 * graph (the pointers and shapes are then frozen into the graph).  The first
 * call on a device sets kernel attributes and queries the device once; make
 * that first call before any stream capture.  Calls are thread-safe.
 *
 * Errors.  Argument faults the host can see return a status and launch
 * nothing.  A failed CUDA call returns MX_ERR_CUDA (mx_last_cuda_error gives
 * the CUDA code).
 * Bad device-side offsets are clamped as stated above.  Every wait of a
 * kernel's copy pipeline has a time limit (about 2^31 SM clocks); a kernel
 * whose wait runs out sets bit 0 of the device flags and returns early, and
 * the output of that call is then undefined (partly written).  The call
 * itself has already returned MX_OK by then: the flags (mx_device_flags) are
 * the only record, and they are shared by every call on the device, so check
 * them after a batch of calls, not per call.
 *
 * Contexts.  The library uses the CUDA context current in the calling
 * thread.  Only when no context is current does it bind the current
 * device's primary context (as the CUDA runtime would); a context the caller
 * made current, primary or not, is left in place.  Kernel attributes (the
 * shared-memory sizes) are set once per device, in the context current at
 * the library's first call on that device: make every call on a device from
 * that same context (normally the primary one).
 */
#ifndef MXSCALE_H
#define MXSCALE_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    MX_OK = 0,
    MX_ERR_INVALID_ARG = 1,  /* null pointer, G outside [1, 64], negative size, stride < cols, sizes too large */
    MX_ERR_MISALIGNED = 2,   /* `out` not 16-byte aligned, or a forced path whose alignment rule fails */
    MX_ERR_UNSUPPORTED = 3,  /* shape beyond the kernels' index range */
    MX_ERR_CUDA = 4          /* a CUDA runtime or driver call failed */
} mx_status;

typedef enum { MX_GROUPS_M = 0, MX_GROUPS_K = 1 } mx_group_dim;

/* Kernel choice.  AUTO takes, in order of preference:
 *   TMA   2-D tensor-map loads: `scales` 16-byte aligned, row stride a multiple of 16;
 *   FLAT  1-D tensor-map loads of whole row blocks (groups along M only): `scales`
 *         16-byte aligned, row stride and cols multiples of 4, row stride <= 256;
 *   WORD  32-bit loads: `scales` and the row stride multiples of 4;
 *   BYTE  byte loads: anything else.
 * Forcing a path whose alignment rule fails returns MX_ERR_MISALIGNED; forcing
 * FLAT for groups along K or a stride above 256 returns MX_ERR_UNSUPPORTED. */
typedef enum { MX_PATH_AUTO = 0, MX_PATH_TMA = 1, MX_PATH_WORD = 2, MX_PATH_BYTE = 3, MX_PATH_FLAT = 4 } mx_path;

#define MX_MAX_GROUPS 64

/* Bytes the caller must allocate for `out`:
 *   M: (rows + 128 * num_groups) * roundup(cols, 4)
 *   K: roundup(rows, 128) * (cols + 4 * num_groups)
 * an upper bound on the padded output for any split of the groups, known on
 * the host without reading the offsets.  Host-only.  Returns 0 for invalid
 * arguments (and for shapes whose allocation is genuinely empty). */
size_t mx_rearranged_size(mx_group_dim dim, int64_t rows, int64_t cols, int32_t num_groups);

/* Groups along M.
 *   scales             device, uint8, element (i, j) at scales[i * row_stride + j];
 *                      any alignment; may be NULL when rows == 0 or cols == 0
 *   rows, cols         >= 0, each at most 2^31 - 2^14
 *   row_stride         bytes between rows, >= cols
 *   group_end_offsets  device, int32[num_groups], cumulative row ends
 *   num_groups         1..64
 *   out                device, 16-byte aligned, mx_rearranged_size(MX_GROUPS_M, ...) bytes,
 *                      must not overlap `scales`
 *   stream             CUDA stream (0 = legacy default stream)
 */
mx_status mx_rearrange_m_groups(const uint8_t *scales, int64_t rows, int64_t cols, int64_t row_stride,
                                const int32_t *group_end_offsets, int32_t num_groups, uint8_t *out,
                                cudaStream_t stream);

/* Groups along K: as mx_rearrange_m_groups, with group_end_offsets holding
 * cumulative scale-column ends and `out` sized by mx_rearranged_size(MX_GROUPS_K, ...). */
mx_status mx_rearrange_k_groups(const uint8_t *scales, int64_t rows, int64_t cols, int64_t row_stride,
                                const int32_t *group_end_offsets, int32_t num_groups, uint8_t *out,
                                cudaStream_t stream);

/* Either dimension with an explicit kernel choice (tests and benchmarks). */
mx_status mx_rearrange_ex(mx_group_dim dim, const uint8_t *scales, int64_t rows, int64_t cols,
                          int64_t row_stride, const int32_t *group_end_offsets, int32_t num_groups,
                          uint8_t *out, mx_path path, cudaStream_t stream);

/* Inverse of mx_rearrange_m_groups: read a blocked buffer (16-byte aligned, laid
 * out as mx_rearrange_m_groups writes it for the same rows, cols and group
 * ends) and write the row-major scales: element (i, j) at
 * scales[i * row_stride + j], any alignment.  Elements that no group covers
 * (rows at or past the last clamped end) are written as 0; bytes between
 * cols and row_stride are not touched.  The values of `blocked`'s padding
 * bytes do not matter (whole tiles are read, padding included, and ignored).
 * Same limits, clamping and stream rules as the forward call; the blocked
 * buffer must not overlap `scales`.  (The other side of the layout
 * the pytorch/ao pages convert to: #3604, 128x4 tiles in each group.) */
mx_status mx_unrearrange_m_groups(const uint8_t *blocked, int64_t rows, int64_t cols,
                                  const int32_t *group_end_offsets, int32_t num_groups, uint8_t *scales,
                                  int64_t row_stride, cudaStream_t stream);

/* Inverse of mx_rearrange_k_groups (groups along columns; uncovered columns
 * at or past the last clamped end are written as 0). */
mx_status mx_unrearrange_k_groups(const uint8_t *blocked, int64_t rows, int64_t cols,
                                  const int32_t *group_end_offsets, int32_t num_groups, uint8_t *scales,
                                  int64_t row_stride, cudaStream_t stream);

/* Padded group starts as the blocked layout uses them (pytorch/ao #3285,
 * Context: the new start of each padded group), for a consumer that would
 * otherwise rescan: starts[g] = sum_{h<g} roundup(n_h, 128) rows (M) or
 * sum_{h<g} roundup(w_h, 4) columns (K), and starts[G] = the padded total.
 * `starts` is device int32[num_groups + 1]; one warp computes it on `stream`
 * from the device offsets (clamped as above).  Group g's blocked bytes start
 * at starts[g] * roundup(cols, 4) (M) or roundup(rows, 128) * starts[g] (K). */
mx_status mx_padded_group_starts(mx_group_dim dim, int64_t rows, int64_t cols, const int32_t *group_end_offsets,
                                 int32_t num_groups, int32_t *starts, cudaStream_t stream);

/* The path AUTO would take for these arguments (host-only, no device access). */
mx_path mx_select_path(mx_group_dim dim, const void *scales, int64_t rows, int64_t cols, int64_t row_stride);

/* Static description of a status code. */
const char *mx_status_string(mx_status status);

/* Device-side error flags of the current device (bit 0: a pipeline wait ran
 * past its time limit and the kernel returned early; the output of the call
 * that set it is undefined).  The flags accumulate over every call of every
 * thread on the device until cleared, so a set bit names no call.
 * Synchronises the device: for tests and debugging, never on a hot path.
 * `clear` != 0 resets the flags after reading. */
mx_status mx_device_flags(uint32_t *flags, int clear);

/* Failure-detection self-test: launches one CTA that waits, with the same
 * bounded mbarrier wait the pipelines use, on a barrier nothing arrives at.
 * The wait gives up after `limit_cycles` SM clocks (1 .. 2^32) and sets bit 0
 * of the device flags; read them with mx_device_flags.  The kernel returns
 * normally and the context stays usable.  Asynchronous on `stream`. */
mx_status mx_selftest_bounded_wait(int64_t limit_cycles, cudaStream_t stream);

/* The CUDA error code behind the calling thread's most recent MX_ERR_CUDA
 * (0 if none): a cudaError_t, or the CUresult of a failed tensor-map encode.  The library reports launch failures from the launch's own
 * return code and never reads or clears the thread's pending CUDA error. */
int mx_last_cuda_error(void);

/* Library version, major * 10000 + minor * 100 + patch. */
int mx_version(void);

#ifdef __cplusplus
}
#endif
#endif /* MXSCALE_H */
