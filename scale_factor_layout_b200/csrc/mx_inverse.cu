// mx_inverse.cu -- the other side of the layout: per-group 128x4 blocked scale
// factors back to row-major, and the padded group starts as a side output.
//
// The blocked layout is the one of mx_rearrange.cu (pytorch/ao #3604: each
// group made of 128x4 scale-factor tiles; #3285: padded group starts are a
// prefix sum of padded sizes, computed in the kernel).  The inverse reads a
// work item's tiles as whole 512-byte lines (one warp reads one tile per
// 128-bit load), transposes 4x4 words in registers, and writes 16-byte row
// segments; the padded starts come from the same warp-shuffle scan.

#include <cuda.h>
#include <cuda_runtime.h>

#include <climits>

#include "mx_device.cuh"
#include "mxscale.h"

// Defined in mx_rearrange.cu: note a CUDA failure for mx_last_cuda_error().
mx_status mx_record_cuda_error(cudaError_t e);

namespace mx {
namespace {

// Shared-memory row block of one work item: 128 rows x 128 columns at pitch
// 176 bytes (11 x 16, odd: conflict-free 16-byte accesses down a column),
// the item's first column 16 bytes into each row so that a window may start
// up to 15 bytes before it.
constexpr int kInvPitch = 176;
constexpr int kInvLead = 16;
constexpr int kInvChunks = 9;   // 16-byte global chunks a 128-column row segment can touch

// One CTA per work item (grid-stride).
//  1. Thread (j = lane, q = warp) loads line j of tiles 4q..4q+3 (a warp reads
//     one whole 512-byte tile per 128-bit load); word a of line j of tile cb
//     holds row j + 32a, columns 4cb .. 4cb+3, so a 4x4 word transpose in
//     registers gives 16 bytes of each of rows j, j+32, j+64, j+96, which go to
//     the shared row block.
//  2. Threads then walk (row, 16-byte-aligned global chunk) pairs: each reads
//     the 32-byte shared window around its chunk, shifts it into place, and
//     stores 16 bytes (or only the bytes of the item at a row's head and tail).
template <bool kDimM>
__global__ void __launch_bounds__(kThreads)
unrearrange_kernel(const uint8_t *__restrict__ blocked, const int32_t *__restrict__ ends,
                   uint8_t *__restrict__ scales, int64_t row_stride, Shape s) {
    __shared__ GroupTable table;
    __shared__ __align__(16) uint8_t rowblk[kTileRows * kInvPitch];
    const int tid = threadIdx.x;
    const int j = tid & 31;
    const int q = tid >> 5;

    grid_dependency_wait();
    if (q == 0) build_group_table<kDimM>(ends, s.G, kDimM ? s.rows : s.cols, s.col_chunks, table);
    __syncthreads();
    const int total = total_items<kDimM>(table, s);

    for (int i = blockIdx.x; i < total; i += gridDim.x) {
        const Item it = decode_item<kDimM>(table, s, i, 1);
        uint4 w[4];
#pragma unroll
        for (int t = 0; t < 4; ++t) {
            const int tile = 4 * q + t;
            w[t] = tile < it.ntiles
                       ? __ldg(reinterpret_cast<const uint4 *>(blocked + it.out_off + (int64_t)tile * 512 + 16 * j))
                       : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int a = 0; a < 4; ++a)
            *reinterpret_cast<uint4 *>(rowblk + (j + 32 * a) * kInvPitch + kInvLead + 16 * q) =
                make_uint4(word_of(w[0], a), word_of(w[1], a), word_of(w[2], a), word_of(w[3], a));
        __syncthreads();

        const int ncol = it.cols_valid;
        const int npairs = it.rows_valid * kInvChunks;
        for (int idx = tid; idx < npairs; idx += kThreads) {
            const int r = idx / kInvChunks;
            const int p = idx - r * kInvChunks;
            uint8_t *row = scales + (int64_t)(it.y + r) * row_stride + it.x;   // item column 0 of row r
            const int lead = (int)(reinterpret_cast<uintptr_t>(row) & 15u);
            // global chunk p covers item columns [16p - lead, 16p - lead + 16)
            const int c0 = 16 * p - lead;
            if (c0 >= ncol) continue;
            const uint8_t *win = rowblk + r * kInvPitch + 16 * p;           // shared bytes [16p, 16p + 32)
            const uint4 lo = *reinterpret_cast<const uint4 *>(win);
            const uint4 hi = *reinterpret_cast<const uint4 *>(win + 16);
            const uint4 v = lead == 0 ? hi : realign(lo, hi, 16 - lead);
            const int kmin = c0 < 0 ? -c0 : 0;
            const int kmax = min(16, ncol - c0);
            uint8_t *dst = row + c0;                                          // 16-byte aligned
            if (kmin == 0 && kmax == 16) {
                *reinterpret_cast<uint4 *>(dst) = v;
            } else {
                const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int k4 = 0; k4 < 4; ++k4) {
                    const int b0 = 4 * k4;
                    if (b0 >= kmin && b0 + 4 <= kmax) {
                        *reinterpret_cast<uint32_t *>(dst + b0) = wv[k4];
                    } else {
                        for (int b = max(b0, kmin); b < min(b0 + 4, kmax); ++b)
                            dst[b] = (uint8_t)(wv[k4] >> (8 * (b - b0)));
                    }
                }
            }
        }
        __syncthreads();
    }

    // Elements no group covers (rows past the last end for M, columns past
    // it for K) are written as zeros; the gaps between rows are not touched.
    const int used = table.begin[s.G - 1] + table.size[s.G - 1];   // E'[G-1]
    const int64_t zr0 = kDimM ? used : 0;
    const int64_t zc0 = kDimM ? 0 : used;
    const int64_t zrows = s.rows - zr0, zcols = s.cols - zc0;
    if (zrows > 0 && zcols > 0) {
        const int64_t n = zrows * zcols;
        const int64_t stride = (int64_t)gridDim.x * blockDim.x;
        for (int64_t k = (int64_t)blockIdx.x * blockDim.x + tid; k < n; k += stride) {
            const int64_t r = zr0 + k / zcols, c = zc0 + k % zcols;
            scales[r * row_stride + c] = 0;
        }
    }
}

// One warp: the padded start of every group (rows for M, columns for K) and
// the padded total, as int32[G + 1].
template <bool kDimM>
__global__ void padded_starts_kernel(const int32_t *__restrict__ ends, int32_t *__restrict__ starts, Shape s) {
    __shared__ GroupTable table;
    grid_dependency_wait();
    build_group_table<kDimM>(ends, s.G, kDimM ? s.rows : s.cols, 1, table);
    __syncwarp();
    for (int g = threadIdx.x; g <= s.G; g += 32) starts[g] = g < s.G ? table.pstart[g] : table.pstart[kMaxGroups];
}

constexpr int64_t kMaxExtent = (1ll << 31) - (1ll << 14);

template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), int grid, int block, cudaStream_t stream, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(block);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

Shape make_shape(int64_t rows, int64_t cols, int32_t G) {
    Shape s;
    s.rows = (int32_t)rows;
    s.cols = (int32_t)cols;
    s.G = G;
    s.padded_cols = (int32_t)(ceil_div(cols, 4) * 4);
    s.padded_rows = (int32_t)(ceil_div(rows, 128) * 128);
    s.col_chunks = (int32_t)ceil_div(s.padded_cols, kChunkCols);
    return s;
}

mx_status unrearrange(mx_group_dim dim, const uint8_t *blocked, int64_t rows, int64_t cols,
                      const int32_t *ends, int32_t G, uint8_t *scales, int64_t row_stride, cudaStream_t stream) {
    if (dim != MX_GROUPS_M && dim != MX_GROUPS_K) return MX_ERR_INVALID_ARG;
    if (G < 1 || G > MX_MAX_GROUPS) return MX_ERR_INVALID_ARG;
    if (rows < 0 || cols < 0 || rows > kMaxExtent || cols > kMaxExtent) return MX_ERR_INVALID_ARG;
    if (row_stride < cols || ends == nullptr) return MX_ERR_INVALID_ARG;
    if (rows == 0 || cols == 0) return MX_OK;   // nothing to write
    if (blocked == nullptr || scales == nullptr) return MX_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(blocked) & 15u) != 0) return MX_ERR_MISALIGNED;
    const bool dim_m = dim == MX_GROUPS_M;
    const Shape s = make_shape(rows, cols, G);
    const int64_t bound = dim_m ? (ceil_div(rows, 128) + G) * s.col_chunks
                                : ceil_div(rows, 128) * (ceil_div(cols, kChunkCols) + G);
    if (bound > INT_MAX) return MX_ERR_UNSUPPORTED;
    int dev = 0, sms = 0;
    if (cudaError_t e = cudaGetDevice(&dev); e != cudaSuccess) return mx_record_cuda_error(e);
    if (cudaError_t e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev); e != cudaSuccess)
        return mx_record_cuda_error(e);
    const int64_t cap = (int64_t)sms * 8 * 4;
    const int grid = (int)(bound < 1 ? 1 : (bound < cap ? bound : cap));
    cudaError_t e = dim_m ? launch_pdl(unrearrange_kernel<true>, grid, kThreads, stream, blocked, ends, scales,
                                       row_stride, s)
                          : launch_pdl(unrearrange_kernel<false>, grid, kThreads, stream, blocked, ends, scales,
                                       row_stride, s);
    return e == cudaSuccess ? MX_OK : mx_record_cuda_error(e);
}

}  // namespace
}  // namespace mx

extern "C" {

mx_status mx_unrearrange_m_groups(const uint8_t *blocked, int64_t rows, int64_t cols,
                                  const int32_t *group_end_offsets, int32_t num_groups, uint8_t *scales,
                                  int64_t row_stride, cudaStream_t stream) {
    return mx::unrearrange(MX_GROUPS_M, blocked, rows, cols, group_end_offsets, num_groups, scales, row_stride,
                           stream);
}

mx_status mx_unrearrange_k_groups(const uint8_t *blocked, int64_t rows, int64_t cols,
                                  const int32_t *group_end_offsets, int32_t num_groups, uint8_t *scales,
                                  int64_t row_stride, cudaStream_t stream) {
    return mx::unrearrange(MX_GROUPS_K, blocked, rows, cols, group_end_offsets, num_groups, scales, row_stride,
                           stream);
}

mx_status mx_padded_group_starts(mx_group_dim dim, int64_t rows, int64_t cols, const int32_t *group_end_offsets,
                                 int32_t num_groups, int32_t *starts, cudaStream_t stream) {
    if (dim != MX_GROUPS_M && dim != MX_GROUPS_K) return MX_ERR_INVALID_ARG;
    if (num_groups < 1 || num_groups > MX_MAX_GROUPS) return MX_ERR_INVALID_ARG;
    if (rows < 0 || cols < 0 || rows > mx::kMaxExtent || cols > mx::kMaxExtent) return MX_ERR_INVALID_ARG;
    if (group_end_offsets == nullptr || starts == nullptr) return MX_ERR_INVALID_ARG;
    const mx::Shape s = mx::make_shape(rows, cols, num_groups);
    cudaError_t e = dim == MX_GROUPS_M
                        ? mx::launch_pdl(mx::padded_starts_kernel<true>, 1, 32, stream, group_end_offsets, starts, s)
                        : mx::launch_pdl(mx::padded_starts_kernel<false>, 1, 32, stream, group_end_offsets, starts, s);
    return e == cudaSuccess ? MX_OK : mx_record_cuda_error(e);
}

}  // extern "C"
