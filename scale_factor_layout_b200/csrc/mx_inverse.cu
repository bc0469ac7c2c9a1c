// mx_inverse.cu -- the other side of the layout: per-group 128x4 blocked scale
// factors back to row-major, and the padded group starts as a side output.
//
// The blocked layout is the one of mx_rearrange.cu (pytorch/ao #3604: each
// group made of 128x4 scale-factor tiles; #3285: padded group starts are a
// prefix sum of padded sizes, computed in the kernel).  The inverse streams a
// work item's tiles into shared memory with a bulk copy, reads them as whole
// 512-byte lines (one warp reads one tile per 128-bit load), transposes 4x4
// words in registers into a shared row block, and writes the output in
// 16-byte aligned chunks that each have exactly one owning item (partial ones
// as byte-masked bulk copies).  Groups along K into an aligned output take
// another kernel, whose work items are 128x128 boxes of the output written
// with one tensor store each.  The padded starts come from the same
// warp-shuffle scan.

#include <cuda.h>
#include <cuda_runtime.h>

#include <climits>
#include <cstring>
#include <mutex>

#include "mx_device.cuh"
#include "mxscale.h"

// Defined in mx_rearrange.cu: note a CUDA failure for mx_last_cuda_error(),
// and encode a 2-D uint8 tensor map over row-major rows.
mx_status mx_record_cuda_error(cudaError_t e);
mx_status mx_encode_rows_map(CUtensorMap *map, const void *base, int64_t width, int64_t rows, int64_t row_stride,
                             uint32_t box_w, uint32_t box_h, CUtensorMapSwizzle swizzle);

namespace mx {
namespace {

// 1-D bulk copy global -> shared (16-byte aligned addresses, bytes a multiple
// of 16), completed on `bar` as transaction bytes.
__device__ __forceinline__ void bulk_load_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
        ::"r"(smem_addr(dst)), "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_addr(bar))
        : "memory");
}

// Bring `bytes` (a multiple of 16) of global memory at a 16-byte aligned
// address into L2 only.
__device__ __forceinline__ void bulk_prefetch_l2(const void *src, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(reinterpret_cast<uint64_t>(src)), "r"(bytes)
                 : "memory");
}

// 2-D tensor store of one box from shared memory (128B-swizzled, 1024-byte
// aligned) at tensor coordinates (x, y); elements outside the tensor are not
// written.  Tracked in the issuing thread's bulk groups.
__device__ __forceinline__ void tma_store_2d(const CUtensorMap *map, const void *src, int x, int y) {
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];"
                 ::"l"(reinterpret_cast<uint64_t>(map)), "r"(smem_addr(src)), "r"(x), "r"(y)
                 : "memory");
}

// Shared-memory row block of one work item: 128 rows of 144 bytes (9 x 16,
// odd: conflict-free 16-byte accesses down a column), which hold up to 36
// tiles' columns (the item's 32 tiles and the quad before them) or, in shift
// mode, the 9 output chunks a row of the item can touch.  In flat mode the
// rows sit back to back instead (row r at r * cols).
constexpr int kInvPreTiles = 4;                                         // quad loaded before an item
constexpr int kInvPitch = (kTilesPerChunk + kInvPreTiles) * 4;          // 144
constexpr int kInvStages = 2;                                           // items in flight per CTA
constexpr int kInvStageBytes = (kTilesPerChunk + kInvPreTiles) * 512;   // 18 KB
constexpr int kInvBlockBytes = kTileRows * kInvPitch;                   // 18 KB
constexpr int kInvSmemBytes = kInvStages * kInvStageBytes + 2 * kInvBlockBytes + 128;
constexpr int kInvTmaSmemBytes = kInvStages * kInvStageBytes + 2 * kInvBlockBytes + 1024;   // 1024-aligned start
// The narrow instance (4 warps) runs flat mode for rows of at most 48 padded
// columns: an item is at most 12 tiles, its rows at most 6 KB together, so 7
// CTAs fit on an SM and about one row block per CTA is resident at once
// (1032 row blocks of a 131072-row input, 1036 CTAs on a B200).
constexpr int kInvNarrowCols = 48;
constexpr int kInvNarrowStageBytes = (kInvNarrowCols / 4) * 512;             // 6 KB
constexpr int kInvNarrowBlockBytes = kTileRows * kInvNarrowCols + 16;        // 6 KB and a chunk's offset
constexpr int kInvNarrowSmemBytes = kInvStages * kInvNarrowStageBytes + 2 * kInvNarrowBlockBytes + 128;
constexpr uint32_t kInvFlagWaitTimeout = 1u;

// Error flags of the inverse kernels (a pipeline wait ran past its limit).
__device__ unsigned int g_inv_flags = 0;

// A work item of the inverse.  Output columns of one row are written by
// whole 16-byte-aligned chunks; a chunk that straddles two items of the same
// run (a group's columns for K, a row's columns for M) belongs to the later
// item, which therefore also loads the quad of tiles just before its own
// (contiguous in the blocked buffer).  Partial chunks remain only where a
// run starts or ends.
struct InvItem {
    int64_t src_off;      // blocked offset of the first tile loaded
    int64_t src2_off;     // merged seam: blocked offset of the previous group's tiles
    int32_t x, y;         // first output column and row of the item
    int32_t rows_valid;   // rows with data
    int32_t ncol;         // item columns with data (<= 128)
    int32_t nload;        // tiles loaded (own, plus the previous quad)
    int32_t pre;          // columns before the item's first one in the stage: 0 or 16
    int32_t last;         // 1 if the item ends its run
    // Shift mode (row stride a multiple of 16, so every row of the item
    // starts at the same offset within a 16-byte chunk):
    int32_t lead;         // byte offset of item column 0 within its 16-byte chunk
    int32_t lo, hi;       // owned bytes [lo, hi) of a row, counted from its first chunk
    int32_t nch;          // 16-byte output chunks per row the item owns a part of (<= 9)
    int32_t partial;      // 1 if a row's first or last owned chunk is partial
    int32_t merge;        // 1 if the item writes the seam chunk before its group whole
    int32_t n2;           // merged seam: tiles of the previous group loaded (<= 4)
    int32_t b0;           // merged seam: byte of the first needed column in the first of them
    int32_t tx;           // >= 0 if the item's owned bytes are exactly one tensor-store box (clipped):
                          // the box's first column in the output tensor map (a multiple of 16)
};

// Groups along K, shift mode: a 16-byte output chunk that holds the seam
// between a group and the next non-empty one (the seam `ls` bytes into the
// chunk, ls != 0) is written whole by the later group's first item when the
// earlier group has the ls columns before the seam within 4 of its tiles and
// the later group fills the rest of the chunk; otherwise both items write
// their part of it (masked).  Both items evaluate this same function.
__device__ __forceinline__ bool seam_whole(int w_prev, int w_next, int ls) {
    return ls != 0 && w_prev >= ls && ((w_prev - ls) & 3) + ls <= 16 && w_next >= 16 - ls;
}

// `out`, `row_stride`: the row-major output, to tell whether an item's first
// column can start mid-chunk (only then is the quad before it needed).
// `map_w`: width of the output tensor map (0 without one), whose column 0 is
// the 16-byte boundary at or below the output's first byte.
template <bool kDimM, bool kTma>
__device__ __forceinline__ InvItem decode_inv(const GroupTable &t, const Shape &s, int i, const uint8_t *out,
                                              int64_t row_stride, int64_t map_w) {
    const Item it = decode_item<kDimM>(t, s, i, 1);
    int k, run, g, rb = 0;   // item's chunk index in its run, the run's column count, group, row band
    if (kDimM) {
        g = find_group(t, s.G, i);
        const int local = i - t.istart[g];
        k = local - (local / s.col_chunks) * s.col_chunks;
        run = s.cols;
    } else {
        const int per_band = t.istart[kMaxGroups];
        rb = i / per_band;
        const int local = i - rb * per_band;
        g = find_group(t, s.G, local);
        k = local - t.istart[g];
        run = t.size[g];
    }
    // every row of the item starts 16-byte aligned: no chunk straddles the
    // item's first column, so nothing before it is needed
    const bool shift = (row_stride & 15) == 0;
    const bool aligned = shift && ((reinterpret_cast<uintptr_t>(out + (int64_t)it.y * row_stride + it.x) & 15u) == 0);
    const bool pre = k > 0 && !aligned;
    InvItem v;
    v.x = it.x;
    v.y = it.y;
    v.rows_valid = it.rows_valid;
    v.ncol = it.cols_valid;
    v.pre = pre ? 4 * kInvPreTiles : 0;
    v.nload = it.ntiles + (pre ? kInvPreTiles : 0);
    v.src_off = it.out_off - (pre ? kInvPreTiles * 512 : 0);
    v.last = kTilesPerChunk * 4 * (k + 1) >= run ? 1 : 0;
    // owned columns as in the store phase; chunk m covers item columns
    // [16m - lead, 16m - lead + 16)
    v.lead = (int)(reinterpret_cast<uintptr_t>(out + (int64_t)it.y * row_stride + it.x) & 15u);
    v.lo = pre ? 0 : v.lead;
    int hi_c = v.last ? v.ncol : kTilesPerChunk * 4 - v.lead;
    v.merge = 0;
    v.n2 = 0;
    v.b0 = 0;
    v.src2_off = 0;
    if (!kDimM && shift) {
        if (k == 0 && v.lead != 0) {
            int gp = g - 1;
            while (gp >= 0 && t.size[gp] == 0) --gp;
            if (gp >= 0 && seam_whole(t.size[gp], t.size[g], v.lead)) {
                const int wp = t.size[gp], Wp = t.pstart[gp + 1] - t.pstart[gp];
                const int t0 = (wp - v.lead) >> 2;
                v.merge = 1;
                v.lo = 0;
                v.n2 = min(kInvPreTiles, Wp / 4 - t0);
                v.b0 = (wp - v.lead) & 3;
                v.src2_off = (int64_t)s.padded_rows * t.pstart[gp] + (int64_t)rb * kTileRows * Wp + 512ll * t0;
            }
        }
        if (v.last) {
            const int ls = (v.lead + v.ncol) & 15;
            int gn = g + 1;
            while (gn < s.G && t.size[gn] == 0) ++gn;
            if (gn < s.G && seam_whole(t.size[g], t.size[gn], ls)) hi_c = v.ncol - ls;
        }
    }
    v.hi = hi_c + v.lead;
    v.nch = (v.hi + 15) >> 4;
    v.partial = ((v.lo & 15) != 0 || (v.hi & 15) != 0) ? 1 : 0;
    // One tensor store writes a 128 x 128 box, clipped at the map's last row
    // and at its right edge (in whole 16-byte units): usable when that is
    // exactly what the item owns.  Groups along M only: for K-groups rows
    // (4 KB apart at the measured sizes) the tensor store was slower than the
    // threads' own stores (15.7 vs 15.0 us at 7168x4096; M-groups 131072x224:
    // 11.4 vs 12.7 us).
    v.tx = -1;
    if (kTma && kDimM && shift && map_w > 0 && v.lo == 0) {
        const int64_t x = (int64_t)it.x + (int64_t)(reinterpret_cast<uintptr_t>(out) & 15u) - v.lead;
        const bool cols_ok = v.hi == kTilesPerChunk * 4 ? x + kTilesPerChunk * 4 <= map_w
                                                        : x + v.hi == map_w && (map_w & 15) == 0;
        const bool rows_ok = v.rows_valid == kTileRows || v.y + v.rows_valid == s.rows;
        if (cols_ok && rows_ok) v.tx = (int)x;
    }
    return v;
}

// 16 bytes starting at byte o of a shared row (o may be negative; bytes
// outside [0, limit) read as zero).
__device__ __forceinline__ uint4 window16(const uint8_t *row, int o, int limit) {
    const uint4 zero = make_uint4(0u, 0u, 0u, 0u);
    const int f = o & ~15;
    const int d = o - f;
    const uint4 lo = (f >= 0 && f < limit) ? *reinterpret_cast<const uint4 *>(row + f) : zero;
    if (d == 0) return lo;
    const uint4 hi = (f + 16 >= 0 && f + 16 < limit) ? *reinterpret_cast<const uint4 *>(row + f + 16) : zero;
    return realign(lo, hi, d);
}

// Store bytes [kmin, kmax) of v at the 16-byte aligned dst.
__device__ __forceinline__ void store16_part(uint8_t *dst, const uint4 &v, int kmin, int kmax) {
    if (kmin == 0 && kmax == 16) {
        *reinterpret_cast<uint4 *>(dst) = v;
        return;
    }
    const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int k4 = 0; k4 < 4; ++k4) {
        const int b0 = 4 * k4;
        if (b0 >= kmin && b0 + 4 <= kmax) {
            *reinterpret_cast<uint32_t *>(dst + b0) = wv[k4];
        } else {
            for (int b = max(b0, kmin); b < min(b0 + 4, kmax); ++b) dst[b] = (uint8_t)(wv[k4] >> (8 * (b - b0)));
        }
    }
}

// Bulk copy of one 16-byte chunk, shared -> global, writing only the bytes
// whose bit is set in `mask` (bit i: byte i); both addresses 16-byte aligned.
__device__ __forceinline__ void bulk_store16_masked(void *gdst, const void *ssrc, uint16_t mask) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group.cp_mask [%0], [%1], 16, %2;"
                 ::"l"(reinterpret_cast<uint64_t>(gdst)), "r"(smem_addr(ssrc)), "h"(mask) : "memory");
}

// Shift mode: write output chunk p of a row whose chunks start at the
// 16-byte aligned `row` and sit at `src` in shared memory; the item owns
// bytes [lo, hi) of the row's chunk span.  Whole chunks are one 128-bit
// store, partial ones one masked bulk copy.
__device__ __forceinline__ void store_chunk_shift(uint8_t *row, const uint8_t *src, int p, int lo, int hi) {
    const int kmin = max(0, lo - 16 * p), kmax = min(16, hi - 16 * p);
    if (kmin >= kmax) return;
    if (kmin == 0 && kmax == 16) {
        *reinterpret_cast<uint4 *>(row + 16 * p) = *reinterpret_cast<const uint4 *>(src + 16 * p);
    } else {
        bulk_store16_masked(row + 16 * p, src + 16 * p, (uint16_t)(((1u << kmax) - 1u) & ~((1u << kmin) - 1u)));
    }
}

constexpr int kModeRows = 0;    // rows start at different offsets within a 16-byte chunk
constexpr int kModeShift = 1;   // row stride a multiple of 16: one offset for all rows of an item
constexpr int kModeFlat = 2;    // rows back to back (stride == cols <= 128), output 4-byte aligned

// Persistent CTAs walk work items round-robin; one thread streams each item's
// tiles (one contiguous, 512-byte aligned span of the blocked buffer) into a
// stage with a 1-D bulk copy completed on an mbarrier, two stages deep.  Word
// a of line j of tile cb holds row j + 32a, columns 4cb .. 4cb+3.  Per item:
//  1. Transpose into one of two shared row blocks.  Thread (j = lane, q =
//     warp) reads line j of a run of tiles (a warp reads one 512-byte tile
//     per instruction), which gives rows j, j+32, j+64, j+96.
//     Shift mode: row chunk m holds exactly the bytes of output chunk m (item
//     columns from 16m - lead); five tile lines and a funnel shift give it,
//     so the store phase moves aligned 16-byte chunks unchanged.  Other
//     modes: quad qq of tiles gives columns 16qq .. 16qq+15 as loaded.
//  2. One barrier: the stage is free (thread 0 refills it) and the other row
//     block is no longer read (each thread first waits until its own bulk
//     copies have read it).
//  3. Output chunks.  A warp writes 4 rows at a time, lane l taking chunk
//     l % 8 of row l / 8 (one 128-bit store covers four contiguous runs), a
//     ninth chunk by the row's first lane.  Shift mode: whole chunks are
//     plain stores, partial ones (where a run starts or ends) masked bulk
//     copies; with kTma (groups along M), an item that owns exactly one
//     128 x 128-byte box had its row block written 128B-swizzled in step 1
//     and thread 0 writes it with one tensor store.  Rows mode: each chunk is
//     shifted into place from the 32-byte window around it, partial ones
//     stored by words and bytes.  Flat mode (rows back to back in memory):
//     the item's rows are one contiguous span and threads take its chunks in
//     order.
// The kernels below instantiate this body: unrearrange_kernel for every mode
// without tensor stores, unrearrange_tma_m_kernel for shift mode along M.
template <bool kDimM, int kWarpsI, bool kTma>
__device__ __forceinline__ void unrearrange_body(const CUtensorMap *omap, int64_t map_w,
                                                 const uint8_t *__restrict__ blocked, int64_t blocked_size,
                                                 const int32_t *__restrict__ ends, uint8_t *__restrict__ scales,
                                                 int64_t row_stride, const Shape &s, int mode) {
    static_assert(kWarpsI == 8 || kWarpsI == 4, "8 warps (every mode) or 4 (narrow flat rows)");
    constexpr bool kNarrow = kWarpsI == 4;
    constexpr int kStageB = kNarrow ? kInvNarrowStageBytes : kInvStageBytes;
    constexpr int kBlockB = kNarrow ? kInvNarrowBlockBytes : kInvBlockBytes;
    constexpr int kPasses = kNarrow ? 1 : 2;   // quads of tiles per thread (at most 3, or 9)
    extern __shared__ uint8_t dyn_smem[];
    // 1024-byte aligned where a row block may be the source of a 128B-swizzled
    // tensor store (stage and row block sizes are multiples of 1 KB)
    constexpr uintptr_t kAlign = kTma ? 1024 : 128;
    uint8_t *stages = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(dyn_smem) + kAlign - 1) & ~(kAlign - 1));
    uint8_t *rowblks = stages + kInvStages * kStageB;
    __shared__ GroupTable table;
    __shared__ __align__(8) uint64_t full[kInvStages];
    __shared__ InvItem items[kInvStages + 1];   // [kInvStages]: the next refill, decoded ahead
    const int tid = threadIdx.x;
    const int j = tid & 31;
    const int q = tid >> 5;
    const uint4 zero = make_uint4(0u, 0u, 0u, 0u);

    if (tid == 0) {
#pragma unroll
        for (int st = 0; st < kInvStages; ++st) mbar_init(&full[st], 1);
        fence_mbar_init();
    }
    // L2 prefetch of the spans this CTA most likely reads first (item i at
    // about 16 KB * i if every item were full); no observable value, so
    // before the dependency wait.
    if (tid == 32) {
        for (int n = 0; n < kInvStages; ++n) {
            constexpr int kSpan = kNarrow ? kStageB : kTilesPerChunk * 512;
            const int64_t off = (int64_t)kSpan * ((int)blockIdx.x + n * (int)gridDim.x);
            if (off + kSpan <= blocked_size) bulk_prefetch_l2(blocked + off, kSpan);
        }
    }
    grid_dependency_wait();
    if (q == 0) build_group_table<kDimM>(ends, s.G, kDimM ? s.rows : s.cols, s.col_chunks, table);
    __syncthreads();
    grid_launch_dependents();
    const int total = total_items<kDimM>(table, s);
    const int bid = blockIdx.x;
    const int n_my = bid < total ? (total - 1 - bid) / (int)gridDim.x + 1 : 0;

    auto decode = [&](int n) {
        return decode_inv<kDimM, kTma>(table, s, bid + n * (int)gridDim.x, scales, row_stride, map_w);
    };
    auto issue = [&](const InvItem &it, int st) {
        items[st] = it;
        const uint32_t bytes = (uint32_t)it.nload * 512u, bytes2 = (uint32_t)it.n2 * 512u;
        mbar_arrive_expect_tx(&full[st], bytes + bytes2);
        bulk_load_g2s(stages + st * kStageB, blocked + it.src_off, bytes, &full[st]);
        // a merged seam's tiles of the previous group, after the item's own (at most 32: no quad before)
        if (bytes2) bulk_load_g2s(stages + st * kStageB + kTilesPerChunk * 512, blocked + it.src2_off, bytes2,
                                  &full[st]);
    };
    if (tid == 0)
        for (int st = 0; st < kInvStages && st < n_my; ++st) issue(decode(st), st);

    for (int n = 0; n < n_my; ++n) {
        const int st = n % kInvStages;
        // The refill of this stage is decoded while its current copy is in
        // flight, so that only the copy itself is issued after the barrier; it
        // waits in shared memory, not in registers held through the transpose.
        const bool refill = tid == 0 && n + kInvStages < n_my;
        if (refill) items[kInvStages] = decode(n + kInvStages);
        const bool ok = mbar_wait_bounded(&full[st], (uint32_t)(n / kInvStages) & 1u);
        InvItem it;
        uint8_t *rowblk = rowblks + (n & 1) * kBlockB;
        if (ok) {
            it = items[st];
            const uint8_t *stage = stages + st * kStageB;
            if (!kNarrow && mode == kModeShift) {
                // Row chunk m: loaded columns from 16m + pre - lead, i.e. from
                // byte sh / 8 of tile 4m + tb.
                const int from = it.pre - it.lead;   // in [-15, 15]
                const int tb = from >> 2;            // floor
                const int sh = (from & 3) * 8;
#pragma unroll
                for (int pass = 0; pass < 2; ++pass) {
                    const int m = q + 8 * pass;      // at most 9 chunks: warp 0 takes the ninth
                    if (m >= it.nch) break;
                    uint4 w[5];
#pragma unroll
                    for (int t = 0; t < 5; ++t) {
                        const int tile = 4 * m + tb + t;
                        w[t] = (tile >= 0 && tile < it.nload && (t < 4 || sh != 0))
                                   ? *reinterpret_cast<const uint4 *>(stage + tile * 512 + 16 * j)
                                   : zero;
                    }
#pragma unroll
                    for (int a = 0; a < 4; ++a) {
                        const uint32_t x0 = word_of(w[0], a), x1 = word_of(w[1], a), x2 = word_of(w[2], a),
                                       x3 = word_of(w[3], a), x4 = word_of(w[4], a);
                        // chunk m of row j + 32a: plain rows at pitch kInvPitch, or the
                        // 128B-swizzled rows of 128 bytes a tensor store reads
                        *reinterpret_cast<uint4 *>((kTma && it.tx >= 0)
                                                       ? rowblk + (j + 32 * a) * 128 + 16 * (m ^ (j & 7))
                                                       : rowblk + (j + 32 * a) * kInvPitch + 16 * m) =
                            make_uint4(funnel(x0, x1, sh), funnel(x1, x2, sh), funnel(x2, x3, sh), funnel(x3, x4, sh));
                    }
                    if (!kDimM && m == 0 && it.merge) {
                        // Seam chunk: bytes [0, lead) are the previous group's last
                        // columns, from its tiles after the item's own in the stage;
                        // this thread just wrote the chunk's other bytes.
#pragma unroll
                        for (int t = 0; t < 4; ++t)
                            w[t] = t < it.n2 ? *reinterpret_cast<const uint4 *>(stage + (kTilesPerChunk + t) * 512 + 16 * j)
                                             : zero;
                        const int sh0 = it.b0 * 8;
                        uint32_t keep[4];   // per word, the bytes below lead
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int nb = min(max(it.lead - 4 * e, 0), 4);
                            keep[e] = nb == 4 ? 0xffffffffu : (1u << (8 * nb)) - 1u;
                        }
#pragma unroll
                        for (int a = 0; a < 4; ++a) {
                            const uint32_t p0 = word_of(w[0], a), p1 = word_of(w[1], a), p2 = word_of(w[2], a),
                                           p3 = word_of(w[3], a);
                            uint4 *dst = reinterpret_cast<uint4 *>((kTma && it.tx >= 0)
                                                                       ? rowblk + (j + 32 * a) * 128 + 16 * (j & 7)
                                                                       : rowblk + (j + 32 * a) * kInvPitch);
                            const uint4 own = *dst;
                            *dst = make_uint4((funnel(p0, p1, sh0) & keep[0]) | (own.x & ~keep[0]),
                                              (funnel(p1, p2, sh0) & keep[1]) | (own.y & ~keep[1]),
                                              (funnel(p2, p3, sh0) & keep[2]) | (own.z & ~keep[2]),
                                              (funnel(p3, 0u, sh0) & keep[3]) | (own.w & ~keep[3]));
                        }
                    }
                }
                // the tensor store or masked bulk copies of the store phase read this row block
                if (it.partial || (kTma && it.tx >= 0)) fence_proxy_async_smem();
            } else {
                const int nquads = (it.nload + 3) / 4;   // at most 9: warp 0 takes the ninth
#pragma unroll
                for (int pass = 0; pass < kPasses; ++pass) {
                    const int qq = q + kWarpsI * pass;
                    if (qq >= nquads) break;
                    uint4 w[4];
#pragma unroll
                    for (int t = 0; t < 4; ++t) {
                        const int tile = 4 * qq + t;
                        w[t] = tile < it.nload ? *reinterpret_cast<const uint4 *>(stage + tile * 512 + 16 * j) : zero;
                    }
#pragma unroll
                    for (int a = 0; a < 4; ++a) {
                        const int r = j + 32 * a;
                        if (!kNarrow && mode == kModeRows) {
                            *reinterpret_cast<uint4 *>(rowblk + r * kInvPitch + 16 * qq) =
                                make_uint4(word_of(w[0], a), word_of(w[1], a), word_of(w[2], a), word_of(w[3], a));
                        } else if (kDimM) {
                            // Flat mode: the item's rows go to the row block as one span that
                            // starts `flead` bytes in (its offset within a 16-byte chunk of the
                            // output, a multiple of 4), so that its output chunks sit 16-byte
                            // aligned; word stores (cols is a multiple of 4), stopping at the
                            // row's end.
                            const int flead =
                                (int)((reinterpret_cast<uintptr_t>(scales) + (uint64_t)it.y * s.cols) & 15u);
                            uint32_t *dst = reinterpret_cast<uint32_t *>(rowblk + flead + r * s.cols) + 4 * qq;
#pragma unroll
                            for (int t = 0; t < 4; ++t)
                                if (16 * qq + 4 * t < s.cols) dst[t] = word_of(w[t], a);
                        }
                    }
                }
                // the bulk copies of the store phase read this row block
                if (kDimM && mode == kModeFlat) fence_proxy_async_smem();
            }
        }
        // this thread's bulk copies of item n - 1 (masked chunks, a tensor store,
        // a flat span) have read their row block, which item n + 1 overwrites
        // after the barrier
        bulk_wait_read<0>();
        if (__syncthreads_or(!ok)) {
            // A copy never completed: flag it, wait (bounded) for the copies
            // still in flight into this CTA's shared memory, and leave.
            if (tid == 0) {
                atomicOr(&g_inv_flags, kInvFlagWaitTimeout);
                for (int m = n; m < n_my && m < n + kInvStages; ++m)
                    mbar_wait_bounded(&full[m % kInvStages], (uint32_t)(m / kInvStages) & 1u);
            }
            return;
        }
        if (refill) issue(items[kInvStages], st);

        const int p = j & 7;
        if (kTma && mode == kModeShift && it.tx >= 0) {
            if (tid == 0) {
                tma_store_2d(omap, rowblk, it.tx, it.y);
                bulk_commit();
            }
        } else if (!kNarrow && mode == kModeShift) {
            // the 16-byte aligned start of row 0's first chunk; the item owns
            // bytes [lo, hi) of each row's chunk span
            uint8_t *base = scales + (int64_t)it.y * row_stride + it.x - it.lead;
            const int lo = it.lo, hi = it.hi;
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int r = 4 * (q + 8 * k) + (j >> 3);
                if (r < it.rows_valid) {
                    uint8_t *row = base + (int64_t)r * row_stride;
                    const uint8_t *src = rowblk + r * kInvPitch;
                    store_chunk_shift(row, src, p, lo, hi);
                    if (p == 0 && it.nch > 8) store_chunk_shift(row, src, 8, lo, hi);
                }
            }
            if (it.partial) bulk_commit();
        } else if (!kNarrow && mode == kModeRows) {
            uint8_t *base = scales + (int64_t)it.y * row_stride + it.x;   // item column 0 of row 0
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int r = 4 * (q + 8 * k) + (j >> 3);
                if (r < it.rows_valid) {
                    uint8_t *row = base + (int64_t)r * row_stride;
                    const int lead = (int)(reinterpret_cast<uintptr_t>(row) & 15u);
                    // owned item columns: from the chunk boundary before column 0 (an item
                    // that continues a run) and up to the next chunk boundary (unless last)
                    const int lo_own = it.pre ? -lead : 0;
                    const int hi_own = it.last ? it.ncol : kTilesPerChunk * 4 - lead;
                    const uint8_t *src = rowblk + r * kInvPitch;
                    const int c0 = 16 * p - lead;
                    const int kmin = max(0, lo_own - c0), kmax = min(16, hi_own - c0);
                    if (kmin < kmax) store16_part(row + c0, window16(src, c0 + it.pre, kInvPitch), kmin, kmax);
                    // A ninth chunk exists only for the last item of a run whose
                    // columns reach past the eighth chunk boundary; the row's first
                    // lane writes it.  Kept out of the store above so that the warp
                    // does not issue a second pass for it.
                    const int c8 = kTilesPerChunk * 4 - lead;
                    if (p == 0 && c8 < hi_own)
                        store16_part(row + c8, window16(src, c8 + it.pre, kInvPitch), 0, min(16, hi_own - c8));
                }
            }
        } else if (kDimM && tid == 0) {
            // Flat mode (groups along M only): the item's output is one span,
            // `lead` bytes into a 16-byte chunk, at the same offset in the row
            // block: whole chunks go out as one bulk copy, a partial first and
            // last chunk as masked copies.
            const int span = it.rows_valid * s.cols;
            uint8_t *chunk0 = scales + (int64_t)it.y * s.cols;   // the item's first byte ...
            const int lead = (int)(reinterpret_cast<uintptr_t>(chunk0) & 15u);
            chunk0 -= lead;                                      // ... and its chunk's start
            const int end = lead + span;
            const int kf0 = lead ? 1 : 0, kf1 = end >> 4;        // whole chunks [kf0, kf1)
            if (kf1 > kf0) bulk_store_s2g(chunk0 + 16 * kf0, rowblk + 16 * kf0, (uint32_t)(kf1 - kf0) * 16u);
            if (lead)
                bulk_store16_masked(chunk0, rowblk, (uint16_t)(((1u << min(16, end)) - 1u) & ~((1u << lead) - 1u)));
            if ((end & 15) && (kf1 > 0 || !lead))
                bulk_store16_masked(chunk0 + 16 * kf1, rowblk + 16 * kf1, (uint16_t)((1u << (end & 15)) - 1u));
            bulk_commit();
        }
    }
    // the bulk copies read shared memory, which must outlive them
    bulk_wait_all();

    // Elements no group covers (rows past the last end for M, columns past
    // it for K) are written as zeros; the gaps between rows are not touched.
    const int used = table.begin[s.G - 1] + table.size[s.G - 1];   // E'[G-1]
    const int64_t zr0 = kDimM ? used : 0;
    const int64_t zc0 = kDimM ? 0 : used;
    const int64_t zrows = s.rows - zr0, zcols = s.cols - zc0;
    if (zrows > 0 && zcols > 0) {
        const int64_t nz = zrows * zcols;
        const int64_t stride = (int64_t)gridDim.x * blockDim.x;
        for (int64_t k = (int64_t)blockIdx.x * blockDim.x + tid; k < nz; k += stride) {
            const int64_t r = zr0 + k / zcols, c = zc0 + k % zcols;
            scales[r * row_stride + c] = 0;
        }
    }
}

template <bool kDimM, int kWarpsI>
__global__ void __launch_bounds__(kWarpsI * 32, kWarpsI == 8 ? 3 : 7)
unrearrange_kernel(const uint8_t *__restrict__ blocked, int64_t blocked_size, const int32_t *__restrict__ ends,
                   uint8_t *__restrict__ scales, int64_t row_stride, Shape s, int mode) {
    unrearrange_body<kDimM, kWarpsI, false>(nullptr, 0, blocked, blocked_size, ends, scales, row_stride, s, mode);
}

// Groups along M in shift mode: items whose owned bytes are one whole box
// are written with one tensor store each.
__global__ void __launch_bounds__(kThreads, 3)
unrearrange_tma_m_kernel(const __grid_constant__ CUtensorMap omap, int64_t map_w, const uint8_t *__restrict__ blocked,
                         int64_t blocked_size, const int32_t *__restrict__ ends, uint8_t *__restrict__ scales,
                         int64_t row_stride, Shape s, int mode) {
    unrearrange_body<true, 8, true>(&omap, map_w, blocked, blocked_size, ends, scales, row_stride, s, mode);
}

// ------------------------------------------------------------------ K-groups, output boxes
// Groups along K into an output whose base is 16-byte aligned and whose row
// stride is a multiple of 16 (the usual case): work items are boxes of the
// OUTPUT, 128 rows x 128 columns, so that each is written with one 2-D tensor
// store and no byte of the output has two writers.  The columns of a box
// belong to one or more groups ("pieces"); a piece's tiles of the box's row
// band are one contiguous span of the blocked buffer (group g's tiles
// (rb, t) at R*Q_g + rb*128*W_g + 512*t), loaded with one bulk copy each into
// the item's stage.  Per 16-byte output chunk of a row (16 consecutive
// columns of one group's row), five consecutive tiles' words and a funnel
// shift give the bytes, as in the shift-mode transpose above; a chunk that
// holds a seam merges the pieces' bytes by column.  Columns no group covers
// are zero.  A box with more pieces than kBoxPieces, or more tiles than a
// stage holds (groups narrower than about 40 columns), reads the same tile
// lines straight from global memory instead, group by group.  Items go in group-major order (the boxes
// whose first column lies in group 0, band after band, then group 1's, ...),
// so that the items in flight read one stretch of the blocked buffer, which
// lets each CTA prefetch its likely first tiles into L2 before its group
// scan.
constexpr int kBoxPieces = 4;
constexpr int kBoxStageTiles = 40;                    // 32 + 1.5 per piece, rounded up
constexpr int kBoxStageBytes = kBoxStageTiles * 512;  // 20 KB
constexpr int kBoxBlockBytes = kTileRows * 128;       // 16 KB, 128B-swizzled rows of 128 bytes
constexpr int kBoxSmemBytes = kInvStages * kBoxStageBytes + 2 * kBoxBlockBytes + 1024;

struct BoxPiece {
    int64_t src;      // blocked offset of the first tile loaded
    int32_t c0, c1;   // output columns [c0, c1) of the piece
    int32_t b;        // the group's first column
    int32_t f;        // first tile of the group loaded (local tile index)
    int32_t ntl;      // tiles loaded
    int32_t s0;       // stage tile holding tile f
};

struct BoxItem {
    int32_t x, y;     // first output column (a multiple of 128) and row
    int32_t ncols;    // columns of the box inside the output (<= 128)
    int32_t np;       // pieces, or -1: read the box's tile lines from global memory
    int32_t rb;       // row band
    int32_t tiles;    // tiles loaded into the stage
    BoxPiece p[kBoxPieces];
};

// The group that holds column c, for 0 <= c < E'[G-1]: the last group whose
// first column is <= c (begin[] is non-decreasing; that group is never an
// empty one, whose successor starts at the same column).
__device__ __forceinline__ int find_group_col(const GroupTable &t, int G, int c) {
    int lo = 0, hi = G;
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (t.begin[mid] <= c) lo = mid; else hi = mid;
    }
    return lo;
}

// Byte offset in the blocked buffer of local tile `tl` of group g in row band rb.
__device__ __forceinline__ int64_t box_src(const GroupTable &t, const Shape &s, int g, int rb, int tl) {
    const int W = t.pstart[g + 1] - t.pstart[g];
    return (int64_t)s.padded_rows * t.pstart[g] + (int64_t)rb * kTileRows * W + 512ll * tl;
}

// The box of row band rb and columns [128 xb, 128 xb + 128): its pieces,
// written in place (shared memory) by the one thread that decodes.
__device__ __forceinline__ void decode_box_at(const GroupTable &t, const Shape &s, int rb, int xb, BoxItem &it) {
    it.rb = rb;
    it.x = xb * 128;
    it.y = it.rb * kTileRows;
    it.ncols = min(128, s.cols - it.x);
    it.np = 0;
    it.tiles = 0;
    const int used = t.begin[s.G - 1] + t.size[s.G - 1];
    const int xend = it.x + it.ncols;
    if (it.x >= used) return;
    for (int g = find_group_col(t, s.G, it.x); g < s.G && t.begin[g] < xend; ++g) {
        if (t.size[g] == 0) continue;
        if (it.np == kBoxPieces) {
            it.np = -1;
            return;
        }
        BoxPiece &p = it.p[it.np];
        p.b = t.begin[g];
        p.c0 = max(it.x, p.b);
        p.c1 = min(xend, p.b + t.size[g]);
        p.f = (p.c0 - p.b) >> 2;
        p.src = box_src(t, s, g, it.rb, p.f);
        p.ntl = ((p.c1 - 1 - p.b) >> 2) - p.f + 1;
        p.s0 = it.tiles;
        it.tiles += p.ntl;
        if (it.tiles > kBoxStageTiles) {
            it.np = -1;
            return;
        }
        ++it.np;
    }
}

// Boxes per row band whose first column lies in group g (ceil(end/128) -
// ceil(begin/128) for a non-empty group), and after the groups a last entry
// for the boxes at or past the last clamped end; bs[g] is the exclusive
// prefix, bs[G + 1] = boxes per band.  Warp 0, lanes holding g and g + 32.
__device__ __forceinline__ void build_box_starts(const GroupTable &t, int G, int nbox, int32_t *bs) {
    const int lane = threadIdx.x & 31;
    auto nb = [&](int g) {
        if (g >= G || t.size[g] == 0) return 0;
        return (t.begin[g] + t.size[g] + 127) / 128 - (t.begin[g] + 127) / 128;
    };
    const int n0 = nb(lane), n1 = nb(lane + 32);
    const int i0 = warp_scan_sum(n0, lane);
    const int top = __shfl_sync(0xffffffffu, i0, 31);
    const int i1 = warp_scan_sum(n1, lane) + top;
    if (lane < G) bs[lane] = i0 - n0;
    if (lane + 32 < G) bs[lane + 32] = i1 - n1;
    if (lane == 31) {
        const int used = t.begin[G - 1] + t.size[G - 1];
        bs[G] = (used + 127) / 128;     // == i1 (boxes that start inside some group)
        bs[G + 1] = nbox;
    }
}

// Work item i in group-major order: the boxes of group 0 (whose first column
// lies in it) band after band, then group 1's, ..., then the boxes past the
// last group.  Items in flight then read one stretch of the blocked buffer.
__device__ __forceinline__ void decode_box(const GroupTable &t, const Shape &s, const int32_t *bs, int bands, int i,
                                           BoxItem &it) {
    const int G = s.G;
    int lo = 0, hi = G + 1;                       // last g in [0, G] with bands * bs[g] <= i
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (bands * bs[mid] <= i) lo = mid; else hi = mid;
    }
    while (lo < G && bs[lo + 1] == bs[lo]) ++lo;  // skip groups without boxes
    const int nb = bs[lo + 1] - bs[lo];
    const int local = i - bands * bs[lo];
    const int rb = local / nb;
    const int first = lo < G ? (t.begin[lo] + 127) / 128 : bs[G];
    decode_box_at(t, s, rb, first + (local - rb * nb), it);
}

__global__ void __launch_bounds__(kThreads, 3)
unrearrange_box_k_kernel(const __grid_constant__ CUtensorMap omap, const uint8_t *__restrict__ blocked,
                         int64_t blocked_size, const int32_t *__restrict__ ends, uint8_t *__restrict__ scales,
                         int64_t row_stride, Shape s) {
    extern __shared__ uint8_t dyn_smem[];
    uint8_t *stages = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(dyn_smem) + 1023) & ~uintptr_t(1023));
    uint8_t *rowblks = stages + kInvStages * kBoxStageBytes;
    __shared__ GroupTable table;
    __shared__ int32_t bstart[kMaxGroups + 2];
    __shared__ __align__(8) uint64_t full[kInvStages];
    __shared__ BoxItem items[kInvStages + 1];   // item n in slot n % (kInvStages + 1)
    const int tid = threadIdx.x;
    const int j = tid & 31;
    const int q = tid >> 5;   // warp q makes output chunk q of every row
    constexpr int kSlots = kInvStages + 1;

    if (tid == 0) {
        tma_prefetch_desc(&omap);
#pragma unroll
        for (int st = 0; st < kInvStages; ++st) mbar_init(&full[st], 1);
        fence_mbar_init();
    }
    // L2 prefetch of the blocked bytes this CTA most likely reads first: in
    // group-major order item i's tiles lie near 16 KB * i (no observable
    // value, so before the dependency wait)
    if (tid == 32) {
        for (int n = 0; n < kInvStages; ++n) {
            const int64_t off = (int64_t)kBoxBlockBytes * ((int)blockIdx.x + n * (int)gridDim.x);
            if (off + kBoxBlockBytes <= blocked_size) bulk_prefetch_l2(blocked + off, kBoxBlockBytes);
        }
    }
    grid_dependency_wait();
    const int nbox = (s.cols + 127) >> 7;
    if (q == 0) {
        build_group_table<false>(ends, s.G, s.cols, 1, table);
        __syncwarp();
        build_box_starts(table, s.G, nbox, bstart);
    }
    __syncthreads();
    grid_launch_dependents();
    const int bands = s.padded_rows / kTileRows;
    const int total = (s.padded_rows / kTileRows) * nbox;
    const int bid = blockIdx.x;
    const int n_my = bid < total ? (total - 1 - bid) / (int)gridDim.x + 1 : 0;
    const int partial_m = (s.cols & 15) ? ((s.cols & 127) >> 4) : -1;   // chunk of the last box cut by cols

    // thread 0: start the copies of item n (slot n % 3) into stage n % 2
    auto issue = [&](int n) {
        const BoxItem &it = items[n % kSlots];
        const int st = n % kInvStages;
        const uint32_t bytes = it.np > 0 ? (uint32_t)it.tiles * 512u : 0u;
        mbar_arrive_expect_tx(&full[st], bytes);
        for (int k = 0; k < it.np; ++k)
            bulk_load_g2s(stages + st * kBoxStageBytes + it.p[k].s0 * 512, blocked + it.p[k].src,
                          (uint32_t)it.p[k].ntl * 512u, &full[st]);
    };
    if (tid == 0)
        for (int n = 0; n < kInvStages && n < n_my; ++n) {
            decode_box(table, s, bstart, bands, bid + n * (int)gridDim.x, items[n]);
            issue(n);
        }

    for (int n = 0; n < n_my; ++n) {
        const int st = n % kInvStages;
        const bool refill = n + kInvStages < n_my;
        // A thread of another warp than thread 0's decodes the refill into the
        // slot that item n - 1 left, so that thread 0's work between two
        // barriers is only the copies it issues.
        if (refill && tid == 32)
            decode_box(table, s, bstart, bands, bid + (n + kInvStages) * (int)gridDim.x, items[(n + kInvStages) % kSlots]);
        const bool ok = mbar_wait_bounded(&full[st], (uint32_t)(n / kInvStages) & 1u);
        uint8_t *rowblk = rowblks + (n & 1) * kBoxBlockBytes;
        // the item's scalars in registers: items[st] is refilled after the barrier
        int ix = 0, iy = 0, incols = 0;
        if (ok) {
            const BoxItem &it = items[n % kSlots];
            ix = it.x;
            iy = it.y;
            incols = it.ncols;
            const uint8_t *stage = stages + st * kBoxStageBytes;
            const int cc0 = it.x + 16 * q;   // first column of this warp's chunk
            uint4 o[4];
#pragma unroll
            for (int a = 0; a < 4; ++a) o[a] = make_uint4(0u, 0u, 0u, 0u);
            int kf = -1;   // the piece that holds all 16 columns of the chunk, if one does
            for (int k = 0; k < it.np; ++k)
                if (it.p[k].c0 <= cc0 && cc0 + 16 <= it.p[k].c1) kf = k;
            if (kf >= 0) {
                // the common case: no seam and no column past the box in the
                // chunk, so every tile line read lies in the piece's loaded run
                // (the fifth only when the chunk starts inside a tile)
                const BoxPiece &p = it.p[kf];
                const int u = cc0 - p.b;
                const int sh = (u & 3) * 8;
                const uint8_t *ln = stage + (p.s0 + (u >> 2) - p.f) * 512 + 16 * j;
                uint4 w[5];
#pragma unroll
                for (int t = 0; t < 4; ++t) w[t] = *reinterpret_cast<const uint4 *>(ln + t * 512);
                w[4] = sh != 0 ? *reinterpret_cast<const uint4 *>(ln + 4 * 512) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
                for (int a = 0; a < 4; ++a) {
                    const uint32_t x0 = word_of(w[0], a), x1 = word_of(w[1], a), x2 = word_of(w[2], a),
                                   x3 = word_of(w[3], a), x4 = word_of(w[4], a);
                    o[a] = make_uint4(funnel(x0, x1, sh), funnel(x1, x2, sh), funnel(x2, x3, sh), funnel(x3, x4, sh));
                }
            } else if (it.np > 0 && cc0 < it.x + it.ncols) {
                for (int k = 0; k < it.np; ++k) {
                    const BoxPiece &p = it.p[k];
                    if (p.c1 <= cc0 || p.c0 >= cc0 + 16) continue;
                    const int u = cc0 - p.b;           // local column of the chunk's byte 0 (may be < 0)
                    const int t0 = u >> 2;             // floor
                    const int sh = (u & 3) * 8;
                    uint4 w[5];
#pragma unroll
                    for (int t = 0; t < 5; ++t) {
                        const int tl = t0 + t - p.f;   // tile within the piece's loaded run
                        w[t] = (tl >= 0 && tl < p.ntl && (t < 4 || sh != 0))
                                   ? *reinterpret_cast<const uint4 *>(stage + (p.s0 + tl) * 512 + 16 * j)
                                   : make_uint4(0u, 0u, 0u, 0u);
                    }
                    // bytes of the chunk that belong to this piece
                    const int k0 = max(p.c0 - cc0, 0), k1 = min(p.c1 - cc0, 16);
                    uint32_t keep[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int lo = min(max(k0 - 4 * e, 0), 4), hi = min(max(k1 - 4 * e, 0), 4);
                        const uint32_t upto_hi = hi == 4 ? 0xffffffffu : (1u << (8 * hi)) - 1u;
                        const uint32_t below_lo = lo == 4 ? 0xffffffffu : (1u << (8 * lo)) - 1u;
                        keep[e] = upto_hi & ~below_lo;
                    }
#pragma unroll
                    for (int a = 0; a < 4; ++a) {
                        const uint32_t x0 = word_of(w[0], a), x1 = word_of(w[1], a), x2 = word_of(w[2], a),
                                       x3 = word_of(w[3], a), x4 = word_of(w[4], a);
                        o[a].x |= funnel(x0, x1, sh) & keep[0];
                        o[a].y |= funnel(x1, x2, sh) & keep[1];
                        o[a].z |= funnel(x2, x3, sh) & keep[2];
                        o[a].w |= funnel(x3, x4, sh) & keep[3];
                    }
                }
            } else if (it.np < 0 && cc0 < it.x + it.ncols) {
                // More, narrower groups than a stage holds: per group that meets
                // the chunk, the same tile lines, shift and column masks as
                // above, read straight from the blocked buffer (a warp reads
                // whole 512-byte tiles).
                const int cend = min(cc0 + 16, it.x + it.ncols);
                for (int g = find_group_col(table, s.G, cc0); g < s.G && table.begin[g] < cend; ++g) {
                    const int b = table.begin[g], wg = table.size[g];
                    if (wg == 0 || b + wg <= cc0) continue;
                    const int u = cc0 - b;              // local column of the chunk's byte 0 (may be < 0)
                    const int t0 = u >> 2;              // floor
                    const int sh = (u & 3) * 8;
                    const int ntg = (wg + 3) >> 2;      // the group's tiles in a row band
                    const uint8_t *lines = blocked + box_src(table, s, g, it.rb, 0) + 16 * j;
                    uint4 w[5];
#pragma unroll
                    for (int t = 0; t < 5; ++t) {
                        const int tl = t0 + t;
                        w[t] = (tl >= 0 && tl < ntg && (t < 4 || sh != 0))
                                   ? __ldg(reinterpret_cast<const uint4 *>(lines + 512 * tl))
                                   : make_uint4(0u, 0u, 0u, 0u);
                    }
                    const int k0 = max(b - cc0, 0), k1 = min(b + wg, cend) - cc0;
                    uint32_t keep[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int lo = min(max(k0 - 4 * e, 0), 4), hi = min(max(k1 - 4 * e, 0), 4);
                        const uint32_t upto_hi = hi == 4 ? 0xffffffffu : (1u << (8 * hi)) - 1u;
                        const uint32_t below_lo = lo == 4 ? 0xffffffffu : (1u << (8 * lo)) - 1u;
                        keep[e] = upto_hi & ~below_lo;
                    }
#pragma unroll
                    for (int a = 0; a < 4; ++a) {
                        const uint32_t x0 = word_of(w[0], a), x1 = word_of(w[1], a), x2 = word_of(w[2], a),
                                       x3 = word_of(w[3], a), x4 = word_of(w[4], a);
                        o[a].x |= funnel(x0, x1, sh) & keep[0];
                        o[a].y |= funnel(x1, x2, sh) & keep[1];
                        o[a].z |= funnel(x2, x3, sh) & keep[2];
                        o[a].w |= funnel(x3, x4, sh) & keep[3];
                    }
                }
            }
#pragma unroll
            for (int a = 0; a < 4; ++a)
                *reinterpret_cast<uint4 *>(rowblk + (j + 32 * a) * 128 + 16 * (q ^ (j & 7))) = o[a];
            fence_proxy_async_smem();
        }
        // the tensor store of item n - 1 has read its row block, which item n + 1 overwrites
        if (tid == 0) bulk_wait_read<0>();
        if (__syncthreads_or(!ok)) {
            if (tid == 0) {
                atomicOr(&g_inv_flags, kInvFlagWaitTimeout);
                for (int m = n; m < n_my && m < n + kInvStages; ++m)
                    mbar_wait_bounded(&full[m % kInvStages], (uint32_t)(m / kInvStages) & 1u);
            }
            return;
        }
        if (tid == 0) {
            if (refill) issue(n + kInvStages);
            // the map ends at the last whole 16-byte chunk of a row and at the last row
            if (ix < (s.cols & ~15)) {
                tma_store_2d(&omap, rowblk, ix, iy);
                bulk_commit();
            }
        }
        if (incols < 128 && partial_m >= 0 && tid < kTileRows) {
            // the chunk that the output's last column cuts, past the map: byte stores
            const int r = tid;
            if (iy + r < s.rows) {
                const uint8_t *src = rowblk + r * 128 + 16 * (partial_m ^ (r & 7));
                uint8_t *dst = scales + (int64_t)(iy + r) * row_stride + ix + 16 * partial_m;
                for (int k = 0; k < (s.cols & 15); ++k) dst[k] = src[k];
            }
        }
    }
    if (tid == 0) bulk_wait_all();
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

// ------------------------------------------------------------------ host side

constexpr int64_t kMaxExtent = (1ll << 31) - (1ll << 14);

// A plain stream-ordered launch, as in mx_rearrange.cu (no programmatic
// stream serialization: it cost time at every switch between kernels).
template <typename... KArgs, typename... Args>
cudaError_t launch_kernel(void (*kernel)(KArgs...), int grid, int block, int smem, cudaStream_t stream,
                          Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(block);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cfg.attrs = nullptr;
    cfg.numAttrs = 0;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

// Per device, once: allow the inverse kernels their shared memory and note
// how many CTAs of them fit on an SM.
constexpr int kMaxDevices = 128;
std::mutex g_inv_mu;
int g_inv_grid[kMaxDevices][4];   // SMs x resident CTAs: 8-warp, narrow, M tensor-store, K box kernel; 0 until set up

enum InvKernel { kInvWide = 0, kInvNarrow = 1, kInvTmaM = 2, kInvBoxK = 3 };

cudaError_t inverse_grid_cap(InvKernel which, int *cap) {
    int dev = 0;
    if (cudaError_t e = cudaGetDevice(&dev); e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_inv_mu);
    if (g_inv_grid[dev][0] == 0) {
        int sms = 0, occ_m = 0, occ_k = 0, occ_n = 0, occ_t = 0, occ_b = 0;
        const cudaError_t steps[] = {
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev),
            cudaFuncSetAttribute(unrearrange_kernel<true, 8>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 kInvSmemBytes),
            cudaFuncSetAttribute(unrearrange_kernel<false, 8>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 kInvSmemBytes),
            cudaFuncSetAttribute(unrearrange_kernel<true, 4>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 kInvNarrowSmemBytes),
            cudaFuncSetAttribute(unrearrange_tma_m_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 kInvTmaSmemBytes),
            cudaFuncSetAttribute(unrearrange_box_k_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 kBoxSmemBytes),
            cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ_m, unrearrange_kernel<true, 8>, kThreads, kInvSmemBytes),
            cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ_k, unrearrange_kernel<false, 8>, kThreads, kInvSmemBytes),
            cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ_n, unrearrange_kernel<true, 4>, 128, kInvNarrowSmemBytes),
            cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ_t, unrearrange_tma_m_kernel, kThreads, kInvTmaSmemBytes),
            cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ_b, unrearrange_box_k_kernel, kThreads, kBoxSmemBytes),
        };
        for (cudaError_t e : steps)
            if (e != cudaSuccess) return e;
        const int occ = occ_m < occ_k ? occ_m : occ_k;
        if (occ < 1 || occ_n < 1 || occ_t < 1 || occ_b < 1 || sms < 1) return cudaErrorInvalidConfiguration;
        g_inv_grid[dev][kInvWide] = sms * occ;
        g_inv_grid[dev][kInvNarrow] = sms * occ_n;
        g_inv_grid[dev][kInvTmaM] = sms * occ_t;
        g_inv_grid[dev][kInvBoxK] = sms * occ_b;
    }
    *cap = g_inv_grid[dev][which];
    return cudaSuccess;
}

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
    // flat mode: rows back to back, one item per row block, whole words
    const int mode = dim_m && row_stride == cols && cols <= kTilesPerChunk * 4 && cols % 4 == 0 &&
                             (reinterpret_cast<uintptr_t>(scales) & 3u) == 0
                         ? kModeFlat
                     : (row_stride & 15) == 0                                                  ? kModeShift
                                                                                                : kModeRows;
    const bool narrow = mode == kModeFlat && s.padded_cols <= kInvNarrowCols;
    const bool tma_m = mode == kModeShift && dim_m;
    // groups along K into a 16-byte aligned output: boxes of the output, one
    // tensor store each (a map over the whole 16-byte chunks of each row)
    const bool box_k = !dim_m && mode == kModeShift && (reinterpret_cast<uintptr_t>(scales) & 15u) == 0 &&
                       cols >= 16 && row_stride < (1ll << 40);
    int cap = 0;
    if (cudaError_t e = inverse_grid_cap(box_k    ? kInvBoxK
                                         : narrow ? kInvNarrow
                                         : tma_m  ? kInvTmaM
                                                  : kInvWide,
                                         &cap);
        e != cudaSuccess)
        return mx_record_cuda_error(e);
    const int64_t box_bound = ceil_div(rows, 128) * ceil_div(cols, 128);
    const int64_t work = box_k ? box_bound : bound;
    const int grid = (int)(work < 1 ? 1 : (work < cap ? work : cap));
    const int64_t blocked_size = (int64_t)mx_rearranged_size(dim, rows, cols, G);
    cudaError_t e;
    if (box_k) {
        CUtensorMap omap;
        std::memset(&omap, 0, sizeof(omap));
        if (mx_status st = mx_encode_rows_map(&omap, scales, cols & ~int64_t(15), rows, row_stride, 128, 128,
                                              CU_TENSOR_MAP_SWIZZLE_128B);
            st != MX_OK)
            return st;
        e = launch_kernel(unrearrange_box_k_kernel, grid, kThreads, kBoxSmemBytes, stream, omap, blocked,
                          blocked_size, ends, scales, row_stride, s);
    } else if (tma_m) {
        // Whole-box items go out as tensor stores: a map over the output from
        // the 16-byte boundary at or below its first byte, as wide as the rows
        // reach (capped at the row stride; items past the cap use plain stores).
        CUtensorMap omap;
        std::memset(&omap, 0, sizeof(omap));
        const int64_t base_off = (int64_t)(reinterpret_cast<uintptr_t>(scales) & 15u);
        const int64_t map_w = cols + base_off < row_stride ? cols + base_off : row_stride;
        if (mx_status st = mx_encode_rows_map(&omap, scales - base_off, map_w, rows, row_stride, 128, 128,
                                              CU_TENSOR_MAP_SWIZZLE_128B);
            st != MX_OK)
            return st;
        e = launch_kernel(unrearrange_tma_m_kernel, grid, kThreads, kInvTmaSmemBytes, stream, omap, map_w, blocked,
                          blocked_size, ends, scales, row_stride, s, mode);
    } else {
        e = narrow  ? launch_kernel(unrearrange_kernel<true, 4>, grid, 128, kInvNarrowSmemBytes, stream, blocked,
                                    blocked_size, ends, scales, row_stride, s, mode)
            : dim_m ? launch_kernel(unrearrange_kernel<true, 8>, grid, kThreads, kInvSmemBytes, stream, blocked,
                                    blocked_size, ends, scales, row_stride, s, mode)
                    : launch_kernel(unrearrange_kernel<false, 8>, grid, kThreads, kInvSmemBytes, stream, blocked,
                                    blocked_size, ends, scales, row_stride, s, mode);
    }
    return e == cudaSuccess ? MX_OK : mx_record_cuda_error(e);
}

}  // namespace
}  // namespace mx

// Read (and optionally clear) the inverse kernels' error flags; part of
// mx_device_flags (C++ linkage, not part of the C ABI).
cudaError_t mx_inverse_flags(unsigned int *flags, int clear) {
    if (cudaError_t e = cudaMemcpyFromSymbol(flags, mx::g_inv_flags, sizeof(*flags)); e != cudaSuccess) return e;
    if (clear) {
        const unsigned int zero = 0;
        if (cudaError_t e = cudaMemcpyToSymbol(mx::g_inv_flags, &zero, sizeof(zero)); e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

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
                        ? mx::launch_kernel(mx::padded_starts_kernel<true>, 1, 32, 0, stream, group_end_offsets, starts, s)
                        : mx::launch_kernel(mx::padded_starts_kernel<false>, 1, 32, 0, stream, group_end_offsets, starts,
                                         s);
    return e == cudaSuccess ? MX_OK : mx_record_cuda_error(e);
}

}  // extern "C"
