// mx_device.cuh -- device-side building blocks of the scale-factor rearrange
// kernels for sm_100a: PTX wrappers (mbarrier, TMA), the per-CTA group scan,
// work-item decoding, and the 4x32 -> 32x4 word transpose that turns 128 rows
// of scales into 512-byte blocked tiles.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace mx {

constexpr int kThreads = 256;         // 8 warps; warp q owns tiles 4q..4q+3 of a chunk
constexpr int kMaxGroups = 64;
constexpr int kTileRows = 128;
constexpr int kChunkCols = 128;       // columns (bytes) of scales per work item
constexpr int kTilesPerChunk = kChunkCols / 4;
constexpr int kPitchSw = 128;         // M path: TMA box 128 B wide, 128B-swizzled rows
constexpr int kPitchPlain = 144;      // K path / fallback: 144 B rows (9 x 16 B, odd => no bank conflicts)
constexpr int kStageBytesM = kTileRows * kPitchSw;      // 16384
constexpr int kStageBytesK = kTileRows * kPitchPlain;   // 18432
constexpr uint32_t kFlagWaitTimeout = 1u;

// ------------------------------------------------------------------ PTX
__device__ __forceinline__ uint32_t smem_addr(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;"
                 ::"r"(smem_addr(bar)), "r"(bytes) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return done != 0;
}

// Wait for an mbarrier phase with a time limit (about 2^31 SM clocks, ~1 s).
// Returns false if the limit passed; the caller records the failure and
// leaves instead of hanging the GPU.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t *bar, uint32_t parity,
                                                  long long limit = (1ll << 31)) {
    if (mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    while (true) {
        for (int i = 0; i < 64; ++i)
            if (mbar_try_wait(bar, parity)) return true;
        if (clock64() - t0 > limit) return false;
    }
}

__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap *map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// Bring a 2-D box into L2 only (no shared memory, no completion to wait for).
__device__ __forceinline__ void tma_prefetch_l2(const CUtensorMap *map, int x, int y) {
    asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global.tile [%0, {%1, %2}];"
                 ::"l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y) : "memory");
}

// 1-D variants: a box of consecutive elements starting at element x.
__device__ __forceinline__ void tma_load_1d(void *dst, const CUtensorMap *map, int x, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.1d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2}], [%3];"
        ::"r"(smem_addr(dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(smem_addr(bar))
        : "memory");
}

__device__ __forceinline__ void tma_prefetch_l2_1d(const CUtensorMap *map, int x) {
    asm volatile("cp.async.bulk.prefetch.tensor.1d.L2.global.tile [%0, {%1}];"
                 ::"l"(reinterpret_cast<uint64_t>(map)), "r"(x) : "memory");
}

// Bring the 128-byte line holding p into L2.
__device__ __forceinline__ void prefetch_l2(const void *p) {
    asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

// 2-D tiled TMA load of one box into shared memory; completion is signalled
// on `bar` as transaction bytes.  x (the column coordinate) must be a
// multiple of 16 for uint8 data.
__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *map, int x, int y, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];"
        ::"r"(smem_addr(dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_addr(bar))
        : "memory");
}

// Bulk asynchronous shared -> global copy (bytes a multiple of 16, both
// addresses 16-byte aligned), tracked per issuing thread in bulk groups.
__device__ __forceinline__ void bulk_store_s2g(void *gdst, const void *ssrc, uint32_t bytes) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;"
                 ::"l"(reinterpret_cast<uint64_t>(gdst)), "r"(smem_addr(ssrc)), "r"(bytes) : "memory");
}

// An L2 policy that marks lines as the first to evict (data written once and
// not read again by this kernel).
__device__ __forceinline__ uint64_t policy_evict_first() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}

// bulk_store_s2g with an L2 cache policy.
__device__ __forceinline__ void bulk_store_s2g_hint(void *gdst, const void *ssrc, uint32_t bytes, uint64_t policy) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group.L2::cache_hint [%0], [%1], %2, %3;"
                 ::"l"(reinterpret_cast<uint64_t>(gdst)), "r"(smem_addr(ssrc)), "r"(bytes), "l"(policy) : "memory");
}

__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }

// Wait until at most N of this thread's bulk groups still read shared memory.
template <int N>
__device__ __forceinline__ void bulk_wait_read() {
    asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}

// Wait until all of this thread's bulk groups have completed.
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// Programmatic dependent launch: wait for the grids this launch depends on
// (a no-op when launched without the attribute), and allow dependents to be
// scheduled.
__device__ __forceinline__ void grid_dependency_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void grid_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// ------------------------------------------------------------------ scan
// Per-group values every CTA derives from the raw end offsets.
struct GroupTable {
    int32_t begin[kMaxGroups];       // clamped first row (M) / column (K)
    int32_t size[kMaxGroups];        // clamped size
    int32_t pstart[kMaxGroups + 1];  // padded start: P_g rows (M) or Q_g columns (K); [G] = total
    int32_t istart[kMaxGroups + 1];  // first work item of the group (M) / first chunk in a row band (K)
};

__device__ __forceinline__ int warp_scan_max(int v, int lane) {
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        int o = __shfl_up_sync(0xffffffffu, v, d);
        if (lane >= d) v = max(v, o);
    }
    return v;
}

__device__ __forceinline__ int warp_scan_sum(int v, int lane) {
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        int o = __shfl_up_sync(0xffffffffu, v, d);
        if (lane >= d) v += o;
    }
    return v;
}

// Warp 0 builds the table: lane l holds groups l and l + 32.  Ends are made
// monotone and bounded (a running max of max(E, 0), capped at `limit`), then
// two exclusive prefix sums give the padded starts and the work-item starts.
//   M: padded size roundup(n, 128); items ceil(n / 128) * col_chunks.
//   K: padded size roundup(w, 4);   items (chunks per row band) ceil(W / 128).
template <bool kDimM>
__device__ __forceinline__ void build_group_table(const int32_t *__restrict__ ends, int G, int limit,
                                                  int col_chunks, GroupTable &t) {
    const int lane = threadIdx.x & 31;
    const int g0 = lane, g1 = lane + 32;
    int e0 = g0 < G ? max(__ldg(ends + g0), 0) : 0;
    int e1 = g1 < G ? max(__ldg(ends + g1), 0) : 0;
    int m0 = warp_scan_max(e0, lane);
    const int top0 = __shfl_sync(0xffffffffu, m0, 31);
    int m1 = max(warp_scan_max(e1, lane), top0);
    const int end0 = min(m0, limit), end1 = min(m1, limit);
    int b0 = __shfl_up_sync(0xffffffffu, end0, 1);
    int b1 = __shfl_up_sync(0xffffffffu, end1, 1);
    const int last0 = __shfl_sync(0xffffffffu, end0, 31);
    if (lane == 0) {
        b0 = 0;
        b1 = last0;
    }
    // groups past G repeat the last end, so they are empty
    const int n0 = end0 - b0, n1 = end1 - b1;
    int p0, p1, i0, i1;
    if (kDimM) {
        p0 = (n0 + 127) & ~127;
        p1 = (n1 + 127) & ~127;
        i0 = (p0 >> 7) * col_chunks;
        i1 = (p1 >> 7) * col_chunks;
    } else {
        p0 = (n0 + 3) & ~3;
        p1 = (n1 + 3) & ~3;
        i0 = (p0 + kChunkCols - 1) / kChunkCols;
        i1 = (p1 + kChunkCols - 1) / kChunkCols;
    }
    const int ps0 = warp_scan_sum(p0, lane);
    const int ptop = __shfl_sync(0xffffffffu, ps0, 31);
    const int ps1 = warp_scan_sum(p1, lane) + ptop;
    const int is0 = warp_scan_sum(i0, lane);
    const int itop = __shfl_sync(0xffffffffu, is0, 31);
    const int is1 = warp_scan_sum(i1, lane) + itop;
    t.begin[g0] = b0;
    t.begin[g1] = b1;
    t.size[g0] = n0;
    t.size[g1] = n1;
    t.pstart[g0] = ps0 - p0;
    t.pstart[g1] = ps1 - p1;
    t.istart[g0] = is0 - i0;
    t.istart[g1] = is1 - i1;
    if (lane == 31) {
        t.pstart[kMaxGroups] = ps1;
        t.istart[kMaxGroups] = is1;
    }
}

// ------------------------------------------------------------------ work items
// One work item: 128 rows x up to 128 columns of one group, written as up to
// 32 consecutive 512-byte tiles.
struct Item {
    int64_t out_off;     // byte offset of the item's first tile in `out`
    int32_t x, y;        // load origin: column (aligned down) and row of scales
    int32_t delta;       // bytes between the aligned column x and the chunk's first column
    int32_t rows_valid;  // rows of the chunk that hold real data
    int32_t cols_valid;  // columns of the chunk that hold real data
    int32_t ntiles;      // tiles the item writes
};

struct Shape {
    int32_t rows, cols, G;
    int32_t col_chunks;  // M: ceil(roundup(cols,4) / 128)
    int32_t padded_cols; // M: roundup(cols, 4)
    int32_t padded_rows; // K: roundup(rows, 128)
};

// Group g with istart[g] <= i < istart[g+1] (istart is non-decreasing,
// istart[0] = 0, and i < istart[G]).
__device__ __forceinline__ int find_group(const GroupTable &t, int G, int i) {
    int lo = 0, hi = G;
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (t.istart[mid] <= i) lo = mid; else hi = mid;
    }
    return lo;
}

// Total work items for the call.
template <bool kDimM>
__device__ __forceinline__ int total_items(const GroupTable &t, const Shape &s) {
    if (kDimM) return t.istart[kMaxGroups];
    return (s.padded_rows / kTileRows) * t.istart[kMaxGroups];
}

// Bytes of `out` covered by real groups (the rest of the allocation is the zero tail).
template <bool kDimM>
__device__ __forceinline__ int64_t covered_bytes(const GroupTable &t, const Shape &s) {
    if (kDimM) return (int64_t)t.pstart[kMaxGroups] * s.padded_cols;
    return (int64_t)s.padded_rows * t.pstart[kMaxGroups];
}

// `align` is the alignment of the load origin x: 16 for TMA, 4 for word
// loads, 1 for byte loads.
template <bool kDimM>
__device__ __forceinline__ Item decode_item(const GroupTable &t, const Shape &s, int i, int align) {
    Item it;
    if (kDimM) {
        const int g = find_group(t, s.G, i);
        const int local = i - t.istart[g];
        const int rb = local / s.col_chunks;
        const int k = local - rb * s.col_chunks;
        it.x = k * kChunkCols;
        it.delta = 0;
        it.y = t.begin[g] + rb * kTileRows;
        it.rows_valid = min(kTileRows, t.size[g] - rb * kTileRows);
        it.cols_valid = min(kChunkCols, s.cols - k * kChunkCols);
        it.ntiles = min(kTilesPerChunk, s.padded_cols / 4 - k * kTilesPerChunk);
        it.out_off = (int64_t)t.pstart[g] * s.padded_cols + (int64_t)rb * kTileRows * s.padded_cols +
                     (int64_t)k * kTilesPerChunk * 512;
    } else {
        const int per_band = t.istart[kMaxGroups];
        const int rb = i / per_band;
        const int local = i - rb * per_band;
        const int g = find_group(t, s.G, local);
        const int k = local - t.istart[g];
        const int col0 = t.begin[g] + k * kChunkCols;
        it.x = col0 & ~(align - 1);
        it.delta = col0 - it.x;
        it.y = rb * kTileRows;
        const int W = t.pstart[g + 1] - t.pstart[g];
        it.rows_valid = min(kTileRows, s.rows - rb * kTileRows);
        it.cols_valid = min(kChunkCols, t.size[g] - k * kChunkCols);
        it.ntiles = min(kTilesPerChunk, W / 4 - k * kTilesPerChunk);
        it.out_off = (int64_t)s.padded_rows * t.pstart[g] + (int64_t)rb * kTileRows * W +
                     (int64_t)k * kTilesPerChunk * 512;
    }
    return it;
}

// ------------------------------------------------------------------ transpose
// Thread (j = lane, q = warp) gathers, for rows j, j+32, j+64, j+96 of the
// chunk, the 16 bytes of columns 16q..16q+15 (tiles 4q..4q+3).  Output line
// j of tile 4q+t is then the four words (w[0].t, w[1].t, w[2].t, w[3].t):
// tile byte (r%32)*16 + (r/32)*4 + c with r = j + 32a.

// 128B-swizzled rows of 128 bytes (TMA SWIZZLE_128B): 16-byte chunk c of row
// r sits at chunk c ^ (r % 8).  Rows j + 32a share r % 8 = j % 8.
__device__ __forceinline__ void read_rows_swizzled(const uint8_t *stage, int j, int q, uint4 (&w)[4]) {
    const int chunk = (q ^ (j & 7)) << 4;
#pragma unroll
    for (int a = 0; a < 4; ++a)
        w[a] = *reinterpret_cast<const uint4 *>(stage + (j + 32 * a) * kPitchSw + chunk);
}

__device__ __forceinline__ uint32_t funnel(uint32_t lo, uint32_t hi, int sh) {
    return __funnelshift_r(lo, hi, sh);
}

// 16 bytes starting `delta` (1..15) bytes into the 32 bytes lo:hi.
__device__ __forceinline__ uint4 realign(uint4 lo, uint4 hi, int delta) {
    const int sh = (delta & 3) * 8;
    uint32_t a, b, c, d, e;
    switch (delta >> 2) {
        case 0: a = lo.x; b = lo.y; c = lo.z; d = lo.w; e = hi.x; break;
        case 1: a = lo.y; b = lo.z; c = lo.w; d = hi.x; e = hi.y; break;
        case 2: a = lo.z; b = lo.w; c = hi.x; d = hi.y; e = hi.z; break;
        default: a = lo.w; b = hi.x; c = hi.y; d = hi.z; e = hi.w; break;
    }
    return make_uint4(funnel(a, b, sh), funnel(b, c, sh), funnel(c, d, sh), funnel(d, e, sh));
}

// Plain rows of kPitchPlain bytes; the chunk's first column sits `delta`
// bytes into each row.
__device__ __forceinline__ void read_rows_plain(const uint8_t *stage, int j, int q, int delta, uint4 (&w)[4]) {
    if (delta == 0) {
#pragma unroll
        for (int a = 0; a < 4; ++a)
            w[a] = *reinterpret_cast<const uint4 *>(stage + (j + 32 * a) * kPitchPlain + 16 * q);
    } else {
#pragma unroll
        for (int a = 0; a < 4; ++a) {
            const uint8_t *row = stage + (j + 32 * a) * kPitchPlain + 16 * q;
            const uint4 lo = *reinterpret_cast<const uint4 *>(row);
            const uint4 hi = *reinterpret_cast<const uint4 *>(row + 16);
            w[a] = realign(lo, hi, delta);
        }
    }
}

// 16 bytes starting `off` bytes into a shared row (off + 32 within the row
// when off is not a multiple of 16).
__device__ __forceinline__ uint4 read16_at(const uint8_t *row, int off) {
    const uint8_t *base = row + (off & ~15);
    const uint4 lo = *reinterpret_cast<const uint4 *>(base);
    if ((off & 15) == 0) return lo;
    const uint4 hi = *reinterpret_cast<const uint4 *>(base + 16);
    return realign(lo, hi, off & 15);
}

// 4 bytes starting `off` bytes into a shared row (off + 8 within the row).
__device__ __forceinline__ uint32_t read4_at(const uint8_t *row, int off) {
    const uint32_t *base = reinterpret_cast<const uint32_t *>(row + (off & ~3));
    return __funnelshift_r(base[0], base[1], (off & 3) * 8);
}

// Index of group g with pstart[g] <= v < pstart[g + 1] (v < pstart[G]).
__device__ __forceinline__ int find_group_pstart(const GroupTable &t, int G, int v) {
    int lo = 0, hi = G;
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (t.pstart[mid] <= v) lo = mid; else hi = mid;
    }
    return lo;
}

__device__ __forceinline__ uint32_t word_of(const uint4 &v, int t) {
    return t == 0 ? v.x : t == 1 ? v.y : t == 2 ? v.z : v.w;
}

// Zero rows past rows_valid and columns past cols_valid, then write output
// line j of each of this warp's tiles that exist (coalesced: one warp stores
// one whole 512-byte tile per instruction).
__device__ __forceinline__ void mask_and_store(const uint4 (&w)[4], const Item &it, int j, int q,
                                               uint8_t *__restrict__ out) {
    uint32_t rm[4];
#pragma unroll
    for (int a = 0; a < 4; ++a) rm[a] = (j + 32 * a < it.rows_valid) ? 0xffffffffu : 0u;
    uint8_t *base = out + it.out_off + 16 * j;
#pragma unroll
    for (int t = 0; t < 4; ++t) {
        const int tile = 4 * q + t;
        if (tile < it.ntiles) {
            const int nv = it.cols_valid - 4 * tile;
            const uint32_t cm = nv >= 4 ? 0xffffffffu : (nv <= 0 ? 0u : ((1u << (8 * nv)) - 1u));
            uint4 o;
            o.x = word_of(w[0], t) & rm[0] & cm;
            o.y = word_of(w[1], t) & rm[1] & cm;
            o.z = word_of(w[2], t) & rm[2] & cm;
            o.w = word_of(w[3], t) & rm[3] & cm;
            *reinterpret_cast<uint4 *>(base + (int64_t)tile * 512) = o;
        }
    }
}

// As mask_and_store, but into a shared-memory staging block laid out exactly
// like the item's output span (tile t at byte 512 t), for a bulk store.
__device__ __forceinline__ void mask_and_stage(const uint4 (&w)[4], const Item &it, int j, int q,
                                               uint8_t *staging) {
    uint32_t rm[4];
#pragma unroll
    for (int a = 0; a < 4; ++a) rm[a] = (j + 32 * a < it.rows_valid) ? 0xffffffffu : 0u;
#pragma unroll
    for (int t = 0; t < 4; ++t) {
        const int tile = 4 * q + t;
        if (tile < it.ntiles) {
            const int nv = it.cols_valid - 4 * tile;
            const uint32_t cm = nv >= 4 ? 0xffffffffu : (nv <= 0 ? 0u : ((1u << (8 * nv)) - 1u));
            uint4 o;
            o.x = word_of(w[0], t) & rm[0] & cm;
            o.y = word_of(w[1], t) & rm[1] & cm;
            o.z = word_of(w[2], t) & rm[2] & cm;
            o.w = word_of(w[3], t) & rm[3] & cm;
            *reinterpret_cast<uint4 *>(staging + tile * 512 + 16 * j) = o;
        }
    }
}

// Zero [from, size) of `out` (from is a multiple of 16), spread over the grid.
__device__ __forceinline__ void zero_tail(uint8_t *__restrict__ out, int64_t from, int64_t size) {
    if (from >= size) return;
    const int64_t nvec = (size - from) / 16;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    uint4 *v = reinterpret_cast<uint4 *>(out + from);
    for (int64_t k = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; k < nvec; k += stride)
        v[k] = make_uint4(0u, 0u, 0u, 0u);
    if (blockIdx.x == 0) {
        const int64_t tail = from + nvec * 16;
        for (int64_t b = tail + threadIdx.x; b < size; b += blockDim.x) out[b] = 0;
    }
}

}  // namespace mx
