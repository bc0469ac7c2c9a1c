/*
 * mx_oracle.c -- plain, slow, single-threaded CPU statement of the per-group
 * 128x4 blocked ("swizzled") layout of MXFP8 E8M0 scale factors.
 *
 * TEST INFRASTRUCTURE ONLY: the test suite, the smoke check and the
 * benchmark's CPU-baseline leg are its only callers.  It shares nothing with
 * the CUDA path.  The arithmetic follows the definition directly, with no
 * blocking, fusion or reordering; see mx_oracle.h for the sources.
 */
#include "mx_oracle.h"

#include <stdlib.h>
#include <string.h>

enum { DIM_M = 0, DIM_K = 1, MAX_GROUPS = 64 };

static int64_t round_up(int64_t x, int64_t a) { return (x + a - 1) / a * a; }

/* Byte of element (r, c) inside one 512-byte tile of 128 rows x 4 columns. */
static int64_t tile_byte(int64_t r, int64_t c) {
    return (r % 32) * 16 + (r / 32) * 4 + c;
}

static int args_ok(int dim, int64_t rows, int64_t cols, int32_t num_groups) {
    if (dim != DIM_M && dim != DIM_K) return 0;
    if (rows < 0 || cols < 0) return 0;
    if (num_groups < 1 || num_groups > MAX_GROUPS) return 0;
    return 1;
}

int64_t oracle_rearranged_size(int dim, int64_t rows, int64_t cols, int32_t num_groups) {
    if (!args_ok(dim, rows, cols, num_groups)) return -1;
    if (dim == DIM_M) return (rows + 128 * (int64_t)num_groups) * round_up(cols, 4);
    return round_up(rows, 128) * (cols + 4 * (int64_t)num_groups);
}

/* Group ends arrive from device memory the host never reads, so they are made
 * monotone and bounded rather than rejected: E'[g] = min(max(E[g], E'[g-1]), T). */
void oracle_clamp_ends(const int32_t *ends, int32_t num_groups, int64_t limit, int64_t *clamped) {
    int64_t prev = 0;
    for (int32_t g = 0; g < num_groups; ++g) {
        int64_t e = ends[g];
        if (e < prev) e = prev;
        if (e > limit) e = limit;
        clamped[g] = e;
        prev = e;
    }
}

/* Padded group starts: a prefix sum of each group's size rounded up to the
 * tile edge along the grouped dimension (128 rows for M, 4 columns for K). */
int oracle_padded_group_starts(int dim, int64_t rows, int64_t cols, const int32_t *ends,
                               int32_t num_groups, int64_t *starts) {
    if (!args_ok(dim, rows, cols, num_groups)) return -1;
    int64_t e[MAX_GROUPS];
    int64_t edge = (dim == DIM_M) ? 128 : 4;
    oracle_clamp_ends(ends, num_groups, dim == DIM_M ? rows : cols, e);
    int64_t begin = 0, acc = 0;
    for (int32_t g = 0; g < num_groups; ++g) {
        starts[g] = acc;
        acc += round_up(e[g] - begin, edge);
        begin = e[g];
    }
    starts[num_groups] = acc;
    return 0;
}

int64_t oracle_read_bytes(int dim, int64_t rows, int64_t cols, const int32_t *ends, int32_t num_groups) {
    if (!args_ok(dim, rows, cols, num_groups)) return -1;
    int64_t e[MAX_GROUPS];
    oracle_clamp_ends(ends, num_groups, dim == DIM_M ? rows : cols, e);
    int64_t used = e[num_groups - 1];
    return dim == DIM_M ? used * cols : rows * used;
}

int64_t oracle_written_bytes(int dim, int64_t rows, int64_t cols, const int32_t *ends, int32_t num_groups) {
    int64_t starts[MAX_GROUPS + 1];
    if (oracle_padded_group_starts(dim, rows, cols, ends, num_groups, starts) != 0) return -1;
    if (dim == DIM_M) return starts[num_groups] * round_up(cols, 4);
    return round_up(rows, 128) * starts[num_groups];
}

/* Where input element (i, j) of group g lands.  M: the group's padded block
 * starts at row P_g of a matrix round_up(cols, 4) wide; l = i - first row.
 * K: the group's own blocked matrix (round_up(rows,128) x W_g) starts at byte
 * round_up(rows,128) * Q_g; l = j - first column. */
static int64_t dest_m(int64_t P_g, int64_t PC, int64_t l, int64_t j) {
    return P_g * PC + (l / 128) * 128 * PC + (j / 4) * 512 + tile_byte(l % 128, j % 4);
}

static int64_t dest_k(int64_t R, int64_t Q_g, int64_t W_g, int64_t i, int64_t l) {
    return R * Q_g + (i / 128) * 128 * W_g + (l / 4) * 512 + tile_byte(i % 128, l % 4);
}

int oracle_rearrange(int dim, const uint8_t *scales, int64_t rows, int64_t cols, int64_t row_stride,
                     const int32_t *ends, int32_t num_groups, uint8_t *out, int64_t out_size) {
    if (!args_ok(dim, rows, cols, num_groups) || row_stride < cols) return -1;
    if (out_size < oracle_rearranged_size(dim, rows, cols, num_groups)) return -1;
    int64_t e[MAX_GROUPS], starts[MAX_GROUPS + 1];
    oracle_clamp_ends(ends, num_groups, dim == DIM_M ? rows : cols, e);
    oracle_padded_group_starts(dim, rows, cols, ends, num_groups, starts);
    memset(out, 0, (size_t)out_size);

    int64_t begin = 0;
    if (dim == DIM_M) {
        int64_t PC = round_up(cols, 4);
        for (int32_t g = 0; g < num_groups; ++g) {
            for (int64_t i = begin; i < e[g]; ++i)
                for (int64_t j = 0; j < cols; ++j)
                    out[dest_m(starts[g], PC, i - begin, j)] = scales[i * row_stride + j];
            begin = e[g];
        }
    } else {
        int64_t R = round_up(rows, 128);
        for (int32_t g = 0; g < num_groups; ++g) {
            int64_t W_g = round_up(e[g] - begin, 4);
            for (int64_t i = 0; i < rows; ++i)
                for (int64_t j = begin; j < e[g]; ++j)
                    out[dest_k(R, starts[g], W_g, i, j - begin)] = scales[i * row_stride + j];
            begin = e[g];
        }
    }
    return 0;
}

int oracle_dest_index(int dim, int64_t rows, int64_t cols, const int32_t *ends, int32_t num_groups,
                      int64_t *dest) {
    if (!args_ok(dim, rows, cols, num_groups)) return -1;
    int64_t e[MAX_GROUPS], starts[MAX_GROUPS + 1];
    oracle_clamp_ends(ends, num_groups, dim == DIM_M ? rows : cols, e);
    oracle_padded_group_starts(dim, rows, cols, ends, num_groups, starts);
    for (int64_t k = 0; k < rows * cols; ++k) dest[k] = -1;

    int64_t begin = 0;
    for (int32_t g = 0; g < num_groups; ++g) {
        if (dim == DIM_M) {
            int64_t PC = round_up(cols, 4);
            for (int64_t i = begin; i < e[g]; ++i)
                for (int64_t j = 0; j < cols; ++j)
                    dest[i * cols + j] = dest_m(starts[g], PC, i - begin, j);
        } else {
            int64_t R = round_up(rows, 128), W_g = round_up(e[g] - begin, 4);
            for (int64_t i = 0; i < rows; ++i)
                for (int64_t j = begin; j < e[g]; ++j)
                    dest[i * cols + j] = dest_k(R, starts[g], W_g, i, j - begin);
        }
        begin = e[g];
    }
    return 0;
}

/* Gather form.  An output byte o is decoded independently of the scatter
 * arithmetic above: find the group whose padded block holds o, split the
 * offset inside that block into (row block, column block, byte t of the
 * tile), and undo the in-tile placement: t = 16*line + 4*a + c holds tile row
 * 32*a + line, tile column c. */
int oracle_decode_at(int dim, int64_t rows, int64_t cols, const int32_t *ends, int32_t num_groups,
                     const int64_t *pos, int64_t npos, int64_t *src_row, int64_t *src_col) {
    if (!args_ok(dim, rows, cols, num_groups)) return -1;
    int64_t e[MAX_GROUPS], starts[MAX_GROUPS + 1];
    oracle_clamp_ends(ends, num_groups, dim == DIM_M ? rows : cols, e);
    oracle_padded_group_starts(dim, rows, cols, ends, num_groups, starts);
    int64_t PC = round_up(cols, 4), R = round_up(rows, 128);
    for (int64_t p = 0; p < npos; ++p) {
        int64_t o = pos[p];
        src_row[p] = -1;
        src_col[p] = -1;
        int64_t begin = 0;
        for (int32_t g = 0; g < num_groups; ++g) {
            int64_t lo, hi, width;
            if (dim == DIM_M) {
                lo = starts[g] * PC;
                hi = starts[g + 1] * PC;
                width = PC;
            } else {
                lo = R * starts[g];
                hi = R * starts[g + 1];
                width = starts[g + 1] - starts[g];
            }
            if (o >= lo && o < hi) {
                int64_t local = o - lo;
                int64_t block_bytes = 128 * width;        /* one row block of the group */
                int64_t rb = local / block_bytes;
                int64_t in_block = local % block_bytes;
                int64_t cb = in_block / 512;
                int64_t t = in_block % 512;
                int64_t line = t / 16, a = (t % 16) / 4, c = t % 4;
                int64_t r = rb * 128 + a * 32 + line;   /* row within the group's padded matrix */
                int64_t k = cb * 4 + c;                  /* column within it */
                if (dim == DIM_M) {
                    if (r < e[g] - begin && k < cols) {
                        src_row[p] = begin + r;
                        src_col[p] = k;
                    }
                } else {
                    if (r < rows && k < e[g] - begin) {
                        src_row[p] = r;
                        src_col[p] = begin + k;
                    }
                }
                break;
            }
            begin = e[g];
        }
    }
    return 0;
}

int oracle_gather_at(int dim, const uint8_t *scales, int64_t rows, int64_t cols, int64_t row_stride,
                     const int32_t *ends, int32_t num_groups, const int64_t *pos, int64_t npos,
                     uint8_t *vals) {
    if (row_stride < cols) return -1;
    int64_t *r = (int64_t *)malloc(sizeof(int64_t) * (size_t)(npos > 0 ? npos : 1));
    int64_t *c = (int64_t *)malloc(sizeof(int64_t) * (size_t)(npos > 0 ? npos : 1));
    if (!r || !c) {
        free(r);
        free(c);
        return -1;
    }
    int rc = oracle_decode_at(dim, rows, cols, ends, num_groups, pos, npos, r, c);
    if (rc == 0)
        for (int64_t p = 0; p < npos; ++p)
            vals[p] = (r[p] < 0) ? 0 : scales[r[p] * row_stride + c[p]];
    free(r);
    free(c);
    return rc;
}

int oracle_inverse(int dim, const uint8_t *out, int64_t out_size, int64_t rows, int64_t cols,
                   const int32_t *ends, int32_t num_groups, uint8_t *scales_out) {
    if (!args_ok(dim, rows, cols, num_groups)) return -1;
    memset(scales_out, 0, (size_t)(rows * cols));
    const int64_t chunk = 4096;
    int64_t pos[4096], r[4096], c[4096];
    for (int64_t base = 0; base < out_size; base += chunk) {
        int64_t n = (out_size - base < chunk) ? out_size - base : chunk;
        for (int64_t p = 0; p < n; ++p) pos[p] = base + p;
        oracle_decode_at(dim, rows, cols, ends, num_groups, pos, n, r, c);
        for (int64_t p = 0; p < n; ++p)
            if (r[p] >= 0) scales_out[r[p] * cols + c[p]] = out[base + p];
    }
    return 0;
}
