/*
 * mx_oracle.h -- plain, slow CPU statement of the per-group blocked layout of
 * MXFP8 E8M0 scale factors.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product library links, includes
 * or calls this code; only the test suite, the package's smoke check and the
 * benchmark's CPU-baseline leg load it.  It shares no code, header, table or
 * helper with the CUDA path.
 *
 * Source of the method (pytorch/ao pull requests):
 *   - "[mxfp8 moe training] compute prefix sum of group sizes inside kernel
 *     intead of precomputing" (#3285), sections Context and Changes: the start
 *     of each padded group is a prefix sum of padded group sizes.
 *   - "[mxfp8 moe training] add bench script for scale conversion to blocked
 *     format kernels for groups along K" (#3604), body: each group is made of
 *     128x4 scale-factor tiles.
 *   - "Add CuTeDSL MXFP8 K-groups scale rearrange kernel" (#4704), review,
 *     "Additional findings": padding is zero; an empty group adds no columns.
 *   - The blocked layout itself: a group's padded matrix is cut into 128x4
 *     tiles, ordered row-block-major then column-block-minor, 512 bytes each;
 *     element (r, c) of a tile sits at byte (r%32)*16 + (r/32)*4 + c.
 *
 * dim: 0 = groups along M (rows), 1 = groups along K (columns).
 * Group ends are clamped: E'[-1] = 0, E'[g] = min(max(E[g], E'[g-1]), T),
 * T = rows (M) or cols (K).
 *
 * Every function here is pinned by the CPU test suite (closed forms, a
 * reshape-chain brute force, a word-transpose reduction, bijection and
 * round-trip invariants, hand-worked positions, and the allocation size
 * implied by the bandwidth tables of #3604 and #4704).
 */
#ifndef MX_ORACLE_H
#define MX_ORACLE_H
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Bytes of the output allocation: M (rows + 128*G) * roundup(cols, 4);
 * K roundup(rows, 128) * (cols + 4*G).  Returns -1 on invalid arguments. */
int64_t oracle_rearranged_size(int dim, int64_t rows, int64_t cols, int32_t num_groups);

/* Clamped group ends, as stated above. */
void oracle_clamp_ends(const int32_t *ends, int32_t num_groups, int64_t limit, int64_t *clamped);

/* Padded start of every group (rows for M, columns for K); starts[G] is the
 * padded total.  Returns 0, or -1 on invalid arguments. */
int oracle_padded_group_starts(int dim, int64_t rows, int64_t cols, const int32_t *ends,
                               int32_t num_groups, int64_t *starts);

/* Exact bytes of real input covered by groups, and of the padded output they
 * occupy (excluding the allocation's zero tail). */
int64_t oracle_read_bytes(int dim, int64_t rows, int64_t cols, const int32_t *ends, int32_t num_groups);
int64_t oracle_written_bytes(int dim, int64_t rows, int64_t cols, const int32_t *ends, int32_t num_groups);

/* Scatter form: zero the whole output, then place every real byte.
 * Returns 0, or -1 on invalid arguments (out_size below the allocation). */
int oracle_rearrange(int dim, const uint8_t *scales, int64_t rows, int64_t cols, int64_t row_stride,
                     const int32_t *ends, int32_t num_groups, uint8_t *out, int64_t out_size);

/* Destination byte of every input element (row-major rows x cols), or -1 for
 * an element no group covers. */
int oracle_dest_index(int dim, int64_t rows, int64_t cols, const int32_t *ends, int32_t num_groups,
                      int64_t *dest);

/* Gather form: decode output byte positions into the input element they hold,
 * or (-1, -1) for padding. */
int oracle_decode_at(int dim, int64_t rows, int64_t cols, const int32_t *ends, int32_t num_groups,
                     const int64_t *pos, int64_t npos, int64_t *src_row, int64_t *src_col);

/* Gather form: the value of the output at the given positions. */
int oracle_gather_at(int dim, const uint8_t *scales, int64_t rows, int64_t cols, int64_t row_stride,
                     const int32_t *ends, int32_t num_groups, const int64_t *pos, int64_t npos,
                     uint8_t *vals);

/* Inverse: read a blocked output back to row-major (rows x cols, dense);
 * elements that no group covers come back as 0. */
int oracle_inverse(int dim, const uint8_t *out, int64_t out_size, int64_t rows, int64_t cols,
                   const int32_t *ends, int32_t num_groups, uint8_t *scales_out);

#ifdef __cplusplus
}
#endif
#endif
