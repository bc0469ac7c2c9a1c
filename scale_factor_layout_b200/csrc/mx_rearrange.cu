// mx_rearrange.cu -- libmxscale: MXFP8 E8M0 scale factors -> per-group 128x4
// blocked layout on B200 (sm_100a).  Kernels and the C ABI of include/mxscale.h.
//
// Two kernels per grouping dimension:
//   * rearrange_tma_m / rearrange_tma_k: persistent CTAs (one wave across the
//     SMs); one thread streams 128-row boxes of scales into a ring of
//     shared-memory stages with 2-D TMA loads completed on mbarriers and
//     writes finished tiles with bulk shared->global copies, while all 8 warps
//     transpose the stages into staging blocks.  Needs the row stride to be a
//     multiple of 16 bytes (the 2-D TMA stride rule named in pytorch/ao
//     #3708, "fallback cuda kernel for when input doesn't meet 2d TMA
//     constraints", Context).
//   * rearrange_flat_tma: M-groups with narrow rows whose stride is a multiple
//     of 4: 1-D TMA boxes over whole row blocks (an 8-warp instance, and a
//     4-warp one for rows of at most 64 padded columns).
//   * rearrange_fallback: work items loaded with ordinary 32-bit (or byte)
//     loads, for any stride or alignment (#3708's fallback).
// Every CTA scans the group ends itself (#3285, "compute prefix sum of group
// sizes inside kernel", Changes), so no launch depends on device data known
// to the host; the grid is sized from an upper bound on the work and CTAs
// past the real work only help zero the allocation's tail (#4704 review,
// "Grid over-provisioning" and "Output is torch.zeros every call").

#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <climits>
#include <mutex>

#include "mx_device.cuh"
#include "mxscale.h"

namespace mx {

// Error flags written by kernels (read back by mx_device_flags).
__device__ unsigned int g_mx_flags = 0;

constexpr int kStages = 2;       // input boxes in flight per CTA (3 CTAs per SM)
constexpr int kOutBuffers = 2;   // output staging blocks per CTA
constexpr int kOutBytes = kTilesPerChunk * 512;

template <bool kDimM>
constexpr int stage_bytes() { return kDimM ? kStageBytesM : kStageBytesK; }

// Dynamic shared memory of the M-groups (true) and K-groups (false) TMA kernels.
template <bool kDimM>
constexpr int tma_smem_bytes() { return kStages * stage_bytes<kDimM>() + kOutBuffers * kOutBytes + 1024; }

// Persistent M-groups TMA kernel.  A work item is 128 rows x 128 columns of
// one group (all columns of a row block in ceil(roundup(cols,4) / 128)
// items), loaded as one 2-D box with 128-byte swizzle.  Per item n of a CTA:
//   1. wait for its input box (stage n % kStages) and read 4 rows x 16 bytes
//      per thread into registers;
//   2. one barrier: the stage and the staging block n % 2 are free, and the
//      staging block of item n-1 is complete;
//   3. thread 0 refills the stage with the TMA load of item n + kStages
//      (decoded while the stage's load was in flight) and then bulk-stores
//      item n-1's tiles (shared -> global, asynchronous);
//   4. every thread writes its masked output lines of item n into staging.
// Loads and stores are both asynchronous copies driven by one thread, so the
// 8 warps only move data between shared memory and registers.
__global__ void __launch_bounds__(kThreads, 2)
rearrange_tma_m(const __grid_constant__ CUtensorMap tmap, const int32_t *__restrict__ ends,
                uint8_t *__restrict__ out, int64_t out_size, Shape s) {
    constexpr int kStageBytes = kStageBytesM;
    extern __shared__ uint8_t dyn_smem[];
    // 128B swizzle needs 1024-byte aligned stage buffers
    uint8_t *stages = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(dyn_smem) + 1023) & ~uintptr_t(1023));
    uint8_t *staging = stages + kStages * kStageBytes;
    __shared__ GroupTable table;
    __shared__ __align__(8) uint64_t full[kStages];
    __shared__ Item items[kStages];

    const int tid = threadIdx.x;
    const int j = tid & 31;
    const int q = tid >> 5;

    if (tid == 0) {
        tma_prefetch_desc(&tmap);
#pragma unroll
        for (int st = 0; st < kStages; ++st) mbar_init(&full[st], 1);
        fence_mbar_init();
    }
    // Warm L2 with the boxes this CTA most likely loads first while the
    // previous kernel drains and before the group scan is known: item i is
    // placed as if no group were padded.  A prefetch has no observable value,
    // so it may run before the dependency wait.
    if (tid == 32) {
        for (int n = 0; n < kStages; ++n) {
            const int i = (int)blockIdx.x + n * (int)gridDim.x;
            const int y = kTileRows * (i / s.col_chunks);
            const int x = kChunkCols * (i % s.col_chunks);
            if (y < s.rows) tma_prefetch_l2(&tmap, x, y);
        }
    }
    // Inputs may come from the previous kernel in the stream; outputs may
    // still be read by it.  No global load or store happens before this point.
    grid_dependency_wait();
    if (q == 0) build_group_table<true>(ends, s.G, s.rows, s.col_chunks, table);
    __syncthreads();
    grid_launch_dependents();

    const int total = total_items<true>(table, s);
    const int bid = blockIdx.x;
    const int n_my = bid < total ? (total - 1 - bid) / (int)gridDim.x + 1 : 0;

    auto decode = [&](int n) { return decode_item<true>(table, s, bid + n * (int)gridDim.x, 16); };
    auto issue = [&](const Item &it, int st) {
        items[st] = it;
        mbar_arrive_expect_tx(&full[st], kStageBytes);
        tma_load_2d(stages + st * kStageBytes, &tmap, it.x, it.y, &full[st]);
    };

    if (tid == 0)
        for (int st = 0; st < kStages && st < n_my; ++st) issue(decode(st), st);

    int64_t prev_off = 0;     // thread 0: output span of the previous item
    uint32_t prev_bytes = 0;
    for (int n = 0; n < n_my; ++n) {
        const int st = n % kStages;
        const uint32_t parity = (uint32_t)(n / kStages) & 1u;
        // Thread 0 decodes the stage's refill while its current load is in
        // flight; after the barrier it issues that load before anything else.
        const bool refill = tid == 0 && n + kStages < n_my;
        Item next;
        if (refill) next = decode(n + kStages);
        const bool ok = mbar_wait_bounded(&full[st], parity);
        uint4 w[4];
        Item it;
        if (ok) {
            it = items[st];
            read_rows_swizzled(stages + st * kStageBytes, j, q, w);
        }
        // the store that last read staging block n % 2 (item n-2) is the only
        // bulk group still outstanding here
        if (tid == 0) bulk_wait_read<0>();
        if (__syncthreads_or(!ok)) {
            // A load never completed: flag it, wait (bounded) for the copies
            // still in flight into this CTA's shared memory, and leave.
            if (tid == 0) {
                atomicOr(&g_mx_flags, kFlagWaitTimeout);
                for (int m = n; m < n_my && m < n + kStages; ++m)
                    mbar_wait_bounded(&full[m % kStages], (uint32_t)(m / kStages) & 1u);
            }
            return;
        }
        if (tid == 0) {
            if (refill) issue(next, st);
            if (n > 0) {
                bulk_store_s2g(out + prev_off, staging + ((n - 1) & 1) * kOutBytes, prev_bytes);
                bulk_commit();
            }
            prev_off = it.out_off;
            prev_bytes = (uint32_t)it.ntiles * 512u;
        }
        mask_and_stage(w, it, j, q, staging + (n & 1) * kOutBytes);
        fence_proxy_async_smem();
    }
    if (n_my > 0) {
        __syncthreads();
        if (tid == 0) {
            bulk_store_s2g(out + prev_off, staging + ((n_my - 1) & 1) * kOutBytes, prev_bytes);
            bulk_commit();
        }
    }
    zero_tail(out, covered_bytes<true>(table, s), out_size);
    if (tid == 0) bulk_wait_all();
}

// K-groups TMA kernel.  A row band (128 rows) of the output holds, group
// after group, each group's roundup(w_g, 4) / 4 tiles: the band's tile
// stream.  A work item is a run of 32 consecutive tiles of that stream, so
// only the band's last item is short, whatever the group sizes.  The 32
// tiles' source columns span at most 128 input columns (a group boundary
// skips back over the previous group's 0..3 padding columns), so one TMA box
// 144 bytes wide, started at the 16-byte boundary below the first column,
// holds the item.  A thread's 4 tiles usually lie in one group and are read
// as one realigned 16-byte run per row; a quad that straddles a group
// boundary reads each tile's 4 bytes on its own.  The item's tiles are
// staged contiguously and written with one bulk store per group piece.
struct KItem {
    int32_t x, y;        // load origin (x a multiple of 16)
    int32_t rows_valid;
    int32_t tau0;        // first tile of the item in the band's tile stream
    int32_t ntiles;
    int32_t g0;          // group of tile tau0
    int32_t rb;          // row band
    int32_t pad;
};

__global__ void __launch_bounds__(kThreads, 2)
rearrange_tma_k(const __grid_constant__ CUtensorMap tmap, const int32_t *__restrict__ ends,
                uint8_t *__restrict__ out, int64_t out_size, Shape s) {
    constexpr int kStageBytes = kStageBytesK;
    extern __shared__ uint8_t dyn_smem[];
    uint8_t *stages = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(dyn_smem) + 1023) & ~uintptr_t(1023));
    uint8_t *staging = stages + kStages * kStageBytes;
    __shared__ GroupTable table;
    __shared__ __align__(8) uint64_t full[kStages];
    __shared__ KItem items[kStages];

    const int tid = threadIdx.x;
    const int j = tid & 31;
    const int q = tid >> 5;

    if (tid == 0) {
        tma_prefetch_desc(&tmap);
#pragma unroll
        for (int st = 0; st < kStages; ++st) mbar_init(&full[st], 1);
        fence_mbar_init();
    }
    // L2 prefetch of the boxes this CTA most likely loads first, placed as if
    // no group were padded (no observable value, so before the wait).
    if (tid == 32) {
        const int per_band = (s.cols + kChunkCols - 1) / kChunkCols;
        for (int n = 0; n < kStages; ++n) {
            const int i = (int)blockIdx.x + n * (int)gridDim.x;
            const int y = kTileRows * (i / per_band);
            const int x = kChunkCols * (i % per_band);
            if (y < s.rows) tma_prefetch_l2(&tmap, x, y);
        }
    }
    grid_dependency_wait();
    if (q == 0) build_group_table<false>(ends, s.G, s.cols, 1, table);
    __syncthreads();
    grid_launch_dependents();

    const int T = table.pstart[kMaxGroups] >> 2;          // tiles per band
    const int per_band = (T + kTilesPerChunk - 1) / kTilesPerChunk;
    const int total = (s.padded_rows / kTileRows) * per_band;
    const int bid = blockIdx.x;
    const int n_my = bid < total ? (total - 1 - bid) / (int)gridDim.x + 1 : 0;

    auto decode = [&](int n) {
        const int i = bid + n * (int)gridDim.x;
        KItem it;
        it.rb = i / per_band;
        it.tau0 = (i - it.rb * per_band) * kTilesPerChunk;
        it.ntiles = min(kTilesPerChunk, T - it.tau0);
        it.g0 = find_group_pstart(table, s.G, 4 * it.tau0);
        const int src0 = table.begin[it.g0] + 4 * it.tau0 - table.pstart[it.g0];
        it.x = src0 & ~15;
        it.y = it.rb * kTileRows;
        it.rows_valid = min(kTileRows, s.rows - it.y);
        it.pad = 0;
        return it;
    };
    auto issue = [&](const KItem &it, int st) {
        items[st] = it;
        mbar_arrive_expect_tx(&full[st], kStageBytes);
        tma_load_2d(stages + st * kStageBytes, &tmap, it.x, it.y, &full[st]);
    };

    // Thread 0 writes the staged tiles of an item, one bulk copy per group
    // piece, marking the lines first to evict from L2 (this kernel does not
    // read its output; 1-2% over the default policy on a B200).
    const uint64_t policy = policy_evict_first();
    auto store_item = [&](const KItem &it, const uint8_t *stg) {
        int g = it.g0;
        for (int t = 0; t < it.ntiles;) {
            const int tau = it.tau0 + t;
            while (table.pstart[g + 1] <= 4 * tau) ++g;
            const int end = min(it.tau0 + it.ntiles, table.pstart[g + 1] >> 2);
            const int W = table.pstart[g + 1] - table.pstart[g];
            const int64_t dst = (int64_t)s.padded_rows * table.pstart[g] + (int64_t)it.rb * kTileRows * W +
                                (int64_t)(tau - (table.pstart[g] >> 2)) * 512;
            bulk_store_s2g_hint(out + dst, stg + t * 512, (uint32_t)(end - tau) * 512u, policy);
            t = end - it.tau0;
            ++g;
        }
        bulk_commit();
    };

    if (tid == 0)
        for (int st = 0; st < kStages && st < n_my; ++st) issue(decode(st), st);

    KItem prev;
    prev.ntiles = 0;
    for (int n = 0; n < n_my; ++n) {
        const int st = n % kStages;
        const uint32_t parity = (uint32_t)(n / kStages) & 1u;
        // the stage's refill is decoded while its current load is in flight
        const bool refill = tid == 0 && n + kStages < n_my;
        KItem next;
        if (refill) next = decode(n + kStages);
        const bool ok = mbar_wait_bounded(&full[st], parity);
        uint4 w[4] = {};
        uint32_t cm[4] = {0u, 0u, 0u, 0u};
        KItem it;
        if (ok) {
            it = items[st];
            const uint8_t *stage = stages + st * kStageBytes;
            const int tl0 = 4 * q;
            if (tl0 < it.ntiles) {
                const int tau = it.tau0 + tl0;
                int g = it.g0;
                while (table.pstart[g + 1] <= 4 * tau) ++g;
                const int last = min(tl0 + 3, it.ntiles - 1);
                const int src = table.begin[g] + 4 * tau - table.pstart[g];
                if (4 * (it.tau0 + last) < table.pstart[g + 1]) {
                    // the quad's tiles are consecutive columns of one group
                    const int gend = table.begin[g] + table.size[g];
#pragma unroll
                    for (int t = 0; t < 4; ++t) {
                        const int nv = tl0 + t < it.ntiles ? gend - (src + 4 * t) : 0;
                        cm[t] = nv >= 4 ? 0xffffffffu : (nv <= 0 ? 0u : ((1u << (8 * nv)) - 1u));
                    }
#pragma unroll
                    for (int a = 0; a < 4; ++a)
                        w[a] = read16_at(stage + (j + 32 * a) * kPitchPlain, src - it.x);
                } else {
                    // the quad crosses into a later group: one tile at a time
                    int gt = g;
#pragma unroll
                    for (int t = 0; t < 4; ++t) {
                        const int tl = tl0 + t;
                        if (tl < it.ntiles) {
                            while (table.pstart[gt + 1] <= 4 * (it.tau0 + tl)) ++gt;
                            const int srct = table.begin[gt] + 4 * (it.tau0 + tl) - table.pstart[gt];
                            const int nv = table.begin[gt] + table.size[gt] - srct;
                            cm[t] = nv >= 4 ? 0xffffffffu : ((1u << (8 * nv)) - 1u);
#pragma unroll
                            for (int a = 0; a < 4; ++a) {
                                const uint32_t v = read4_at(stage + (j + 32 * a) * kPitchPlain, srct - it.x);
                                if (t == 0) w[a].x = v; else if (t == 1) w[a].y = v; else if (t == 2) w[a].z = v; else w[a].w = v;
                            }
                        }
                    }
                }
            }
        }
        if (tid == 0) bulk_wait_read<0>();
        if (__syncthreads_or(!ok)) {
            if (tid == 0) {
                atomicOr(&g_mx_flags, kFlagWaitTimeout);
                for (int m = n; m < n_my && m < n + kStages; ++m)
                    mbar_wait_bounded(&full[m % kStages], (uint32_t)(m / kStages) & 1u);
            }
            return;
        }
        if (tid == 0) {
            if (refill) issue(next, st);
            if (n > 0) store_item(prev, staging + ((n - 1) & 1) * kOutBytes);
            prev = it;
        }
        // masked lines of this thread's tiles into staging block n % 2
        {
            uint8_t *stg = staging + (n & 1) * kOutBytes;
            uint32_t rm[4];
#pragma unroll
            for (int a = 0; a < 4; ++a) rm[a] = (j + 32 * a < it.rows_valid) ? 0xffffffffu : 0u;
#pragma unroll
            for (int t = 0; t < 4; ++t) {
                const int tl = 4 * q + t;
                if (tl < it.ntiles) {
                    uint4 o;
                    o.x = word_of(w[0], t) & rm[0] & cm[t];
                    o.y = word_of(w[1], t) & rm[1] & cm[t];
                    o.z = word_of(w[2], t) & rm[2] & cm[t];
                    o.w = word_of(w[3], t) & rm[3] & cm[t];
                    *reinterpret_cast<uint4 *>(stg + tl * 512 + 16 * j) = o;
                }
            }
        }
        fence_proxy_async_smem();
    }
    if (n_my > 0) {
        __syncthreads();
        if (tid == 0) store_item(prev, staging + ((n_my - 1) & 1) * kOutBytes);
    }
    zero_tail(out, (int64_t)s.padded_rows * table.pstart[kMaxGroups], out_size);
    if (tid == 0) bulk_wait_all();
}

// Flat-row TMA kernel (groups along M) for narrow rows whose stride is a
// multiple of 4 but not of 16 bytes (e.g. 44 columns), where a 2-D tensor map
// cannot be built.  The scales are viewed as one 1-D array of 32-bit words;
// an item is a whole 128-row block of a group, which spans
// delta + rows * row_stride consecutive bytes, loaded as 1 KB boxes from the
// 16-byte boundary at or below its first byte (boxes past the array's end
// read zeros).  Rows sit at pitch row_stride in shared memory; with the
// stride a multiple of 4 every row starts on a word, and the transpose reads
// 32-bit words.  The pipeline follows rearrange_tma_m.  An item's output is
// one contiguous span of whole tiles, so a warp can write its tiles' lines
// straight from registers with 16-byte stores that cover whole 512-byte
// tiles (kDirect), or stage them for one bulk copy per item as
// rearrange_tma_m does.
//
// Instances: 8 warps, 2 stages and direct stores for rows of more than 64
// padded columns (no staging blocks and two stages, so up to four times the
// CTAs per SM of four stages with staging: 131072x100 7.2 vs 9.8 us,
// 131072x200 10.3 vs 18.1, 1048576x200 72 vs 108 on a B200); 4 warps and 2
// stages for rows of at most 64 (one quad
// of tiles per warp), small enough per CTA that about one row block per CTA
// is resident at once (1032 row blocks of a 131072-row input).  The 4-warp
// kernel stores directly when the items fit in two waves of the grid (the
// store leaves the critical path of a CTA's one or two items: 5-8% faster
// up to 262144 rows of 44 columns) and stages bulk copies otherwise (3-5%
// faster from 524288 rows, where each CTA streams several items).
constexpr int kFlatBoxWords = 256;
constexpr int kFlatBoxBytes = kFlatBoxWords * 4;
constexpr int kFlatStages = 2;
constexpr int kFlatMaxStride = 256;
constexpr int kFlatNarrowCols = 64;   // padded columns up to which the 4-warp instance runs

struct FlatShape {
    int32_t row_stride;     // bytes, a multiple of 4
    int32_t stage_bytes;    // boxes per stage * 1 KB
    int32_t staging_bytes;  // tiles per row block * 512, rounded to 1 KB (staged instances only)
};

template <int kWarpsF, int kStagesF, bool kDirect>
__global__ void __launch_bounds__(kWarpsF * 32)
rearrange_flat_tma(const __grid_constant__ CUtensorMap tmap, const int32_t *__restrict__ ends,
                   uint8_t *__restrict__ out, int64_t out_size, Shape s, FlatShape f) {
    static_assert(kWarpsF == 8 || kWarpsF == 4, "8 warps (up to 16 quads of tiles) or 4 (up to 4)");
    constexpr int kPasses = kWarpsF == 8 ? 2 : 1;   // quads of tiles per thread
    extern __shared__ uint8_t dyn_smem[];
    uint8_t *stages = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(dyn_smem) + 127) & ~uintptr_t(127));
    uint8_t *staging = stages + kStagesF * f.stage_bytes;
    __shared__ GroupTable table;
    __shared__ __align__(8) uint64_t full[kStagesF];
    __shared__ Item items[kStagesF];

    const int tid = threadIdx.x;
    const int j = tid & 31;
    const int q = tid >> 5;
    const int L = f.row_stride;
    const int ntiles = s.padded_cols / 4;     // every item covers all columns
    const int nquads = (ntiles + 3) / 4;

    if (tid == 0) {
        tma_prefetch_desc(&tmap);
#pragma unroll
        for (int st = 0; st < kStagesF; ++st) mbar_init(&full[st], 1);
        fence_mbar_init();
    }
    // L2 prefetch of the row blocks this CTA most likely takes first (row
    // block i if no group were padded); no observable value, so before the wait.
    if (tid == 32) {
        for (int n = 0; n < kStagesF; ++n) {
            const int64_t y = (int64_t)kTileRows * ((int)blockIdx.x + n * (int)gridDim.x);
            if (y >= s.rows) break;
            const int64_t w0 = ((y * L) >> 4) << 2;
            for (int b = 0; b * kFlatBoxBytes < kTileRows * L; ++b)
                tma_prefetch_l2_1d(&tmap, (int)(w0 + b * kFlatBoxWords));
        }
    }
    grid_dependency_wait();
    if (q == 0) build_group_table<true>(ends, s.G, s.rows, 1, table);
    __syncthreads();
    grid_launch_dependents();

    const int total = table.istart[kMaxGroups];
    const int bid = blockIdx.x;
    const int n_my = bid < total ? (total - 1 - bid) / (int)gridDim.x + 1 : 0;

    auto decode = [&](int n) {
        const int i = bid + n * (int)gridDim.x;
        const int g = find_group(table, s.G, i);
        const int rb = i - table.istart[g];
        Item it;
        it.y = table.begin[g] + rb * kTileRows;
        it.rows_valid = min(kTileRows, table.size[g] - rb * kTileRows);
        it.cols_valid = s.cols;
        it.ntiles = ntiles;
        it.out_off = ((int64_t)table.pstart[g] + (int64_t)rb * kTileRows) * s.padded_cols;
        const int64_t byte0 = (int64_t)it.y * L;
        const int64_t word0 = (byte0 >> 4) << 2;
        it.delta = (int)(byte0 - word0 * 4);
        it.x = (int)word0;
        return it;
    };
    auto issue = [&](const Item &it, int st) {
        const int nbox = (it.delta + it.rows_valid * L + kFlatBoxBytes - 1) / kFlatBoxBytes;
        items[st] = it;
        mbar_arrive_expect_tx(&full[st], (uint32_t)nbox * kFlatBoxBytes);
        for (int b = 0; b < nbox; ++b)
            tma_load_1d(stages + st * f.stage_bytes + b * kFlatBoxBytes, &tmap, it.x + b * kFlatBoxWords, &full[st]);
    };

    if (tid == 0)
        for (int st = 0; st < kStagesF && st < n_my; ++st) issue(decode(st), st);

    int64_t prev_off = 0;
    uint32_t prev_bytes = 0;
    for (int n = 0; n < n_my; ++n) {
        const int st = n % kStagesF;
        const uint32_t parity = (uint32_t)(n / kStagesF) & 1u;
        // the stage's refill is decoded while its current load is in flight
        const bool refill = tid == 0 && n + kStagesF < n_my;
        Item next;
        if (refill) next = decode(n + kStagesF);
        const bool ok = mbar_wait_bounded(&full[st], parity);
        Item it;
        uint32_t wv[kPasses][4][4];   // [quad pass][row a][word t]
        if (ok) {
            it = items[st];
            const uint8_t *stage = stages + st * f.stage_bytes + it.delta;
#pragma unroll
            for (int p = 0; p < kPasses; ++p) {
                const int qq = q + kWarpsF * p;
#pragma unroll
                for (int a = 0; a < 4; ++a) {
                    const uint32_t *row = reinterpret_cast<const uint32_t *>(stage + (j + 32 * a) * L) + 4 * qq;
#pragma unroll
                    for (int t = 0; t < 4; ++t) wv[p][a][t] = (qq < nquads) ? row[t] : 0u;
                }
            }
        }
        if (!kDirect && tid == 0) bulk_wait_read<0>();
        if (__syncthreads_or(!ok)) {
            if (tid == 0) {
                atomicOr(&g_mx_flags, kFlagWaitTimeout);
                for (int m = n; m < n_my && m < n + kStagesF; ++m)
                    mbar_wait_bounded(&full[m % kStagesF], (uint32_t)(m / kStagesF) & 1u);
            }
            return;
        }
        if (tid == 0) {
            if (refill) issue(next, st);
            if (!kDirect) {
                if (n > 0) {
                    bulk_store_s2g(out + prev_off, staging + ((n - 1) & 1) * f.staging_bytes, prev_bytes);
                    bulk_commit();
                }
                prev_off = it.out_off;
                prev_bytes = (uint32_t)it.ntiles * 512u;
            }
        }
        // the item's tiles: straight to the output, or into staging block n % 2
        uint8_t *stg = kDirect ? out + it.out_off : staging + (n & 1) * f.staging_bytes;
#pragma unroll
        for (int p = 0; p < kPasses; ++p) {
            const int qq = q + kWarpsF * p;
#pragma unroll
            for (int t = 0; t < 4; ++t) {
                const int tile = 4 * qq + t;
                if (qq < nquads && tile < ntiles) {
                    // columns 4*tile.. are all real (cols is a multiple of 4 here)
                    uint4 o;
                    o.x = (j < it.rows_valid) ? wv[p][0][t] : 0u;
                    o.y = (j + 32 < it.rows_valid) ? wv[p][1][t] : 0u;
                    o.z = (j + 64 < it.rows_valid) ? wv[p][2][t] : 0u;
                    o.w = (j + 96 < it.rows_valid) ? wv[p][3][t] : 0u;
                    *reinterpret_cast<uint4 *>(stg + tile * 512 + 16 * j) = o;
                }
            }
        }
        if (!kDirect) fence_proxy_async_smem();
    }
    if (!kDirect && n_my > 0) {
        __syncthreads();
        if (tid == 0) {
            bulk_store_s2g(out + prev_off, staging + ((n_my - 1) & 1) * f.staging_bytes, prev_bytes);
            bulk_commit();
        }
    }
    zero_tail(out, (int64_t)table.pstart[kMaxGroups] * s.padded_cols, out_size);
    if (tid == 0) bulk_wait_all();
}

// Fallback for any stride and alignment.  One work item per loop trip: every
// thread first issues all of its loads for the item (up to kMaxWordsPerThread
// 32-bit words, or their bytes), then parks them in shared memory; the
// transpose and stores match the TMA kernel's.
constexpr int kMaxWordsPerRow = (3 + kChunkCols + 3) / 4;   // chunk may start 3 bytes into a word
constexpr int kMaxWordsPerThread = (kTileRows * kMaxWordsPerRow + kThreads - 1) / kThreads;

template <bool kDimM, bool kWord>
__global__ void __launch_bounds__(kThreads)
rearrange_fallback(const uint8_t *__restrict__ scales, int64_t row_stride, const int32_t *__restrict__ ends,
                   uint8_t *__restrict__ out, int64_t out_size, Shape s) {
    __shared__ __align__(16) uint8_t stage[kStageBytesK];
    __shared__ GroupTable table;
    const int tid = threadIdx.x;
    const int j = tid & 31;
    const int q = tid >> 5;

    // L2 prefetch of the rows this CTA most likely handles first (M: item i
    // is row block i / col_chunks if no group were padded), before the wait.
    if (kDimM && s.cols <= kChunkCols) {
        const int64_t y = (int64_t)kTileRows * blockIdx.x;
        const int64_t span = (int64_t)kTileRows * row_stride;
        const int64_t off = (int64_t)tid * 128;
        const int64_t extent = (int64_t)(s.rows - 1) * row_stride + s.cols;   // bytes the view spans
        if (y < s.rows && off < span && y * row_stride + off < extent)
            prefetch_l2(scales + y * row_stride + off);
    }
    grid_dependency_wait();
    if (q == 0) build_group_table<kDimM>(ends, s.G, kDimM ? s.rows : s.cols, s.col_chunks, table);
    __syncthreads();
    const int total = total_items<kDimM>(table, s);

    for (int i = blockIdx.x; i < total; i += gridDim.x) {
        const Item it = decode_item<kDimM>(table, s, i, kWord ? 4 : 1);
        // stage row r holds the chunk's bytes from column it.x on, in words
        const int nw = (it.delta + it.cols_valid + 3) >> 2;
        const int dr = kThreads / nw, dw = kThreads - dr * nw;   // (row, word) step per trip
        const int r0 = tid / nw, w0 = tid - r0 * nw;
        uint32_t v[kMaxWordsPerThread];
        {
            int r = r0, w = w0;
#pragma unroll
            for (int u = 0; u < kMaxWordsPerThread; ++u) {
                v[u] = 0;
                if (r < it.rows_valid) {
                    const int gcol = it.x + 4 * w;
                    const uint8_t *src = scales + (int64_t)(it.y + r) * row_stride + gcol;
                    if (kWord && gcol + 4 <= s.cols) {
                        v[u] = __ldg(reinterpret_cast<const uint32_t *>(src));
                    } else {
#pragma unroll
                        for (int b = 0; b < 4; ++b)
                            if (gcol + b < s.cols) v[u] |= (uint32_t)__ldg(src + b) << (8 * b);
                    }
                }
                r += dr;
                w += dw;
                if (w >= nw) { w -= nw; ++r; }
            }
        }
        {
            int r = r0, w = w0;
#pragma unroll
            for (int u = 0; u < kMaxWordsPerThread; ++u) {
                if (r < it.rows_valid) *reinterpret_cast<uint32_t *>(stage + r * kPitchPlain + 4 * w) = v[u];
                r += dr;
                w += dw;
                if (w >= nw) { w -= nw; ++r; }
            }
        }
        __syncthreads();
        uint4 w4[4];
        read_rows_plain(stage, j, q, it.delta, w4);
        mask_and_store(w4, it, j, q, out);
        __syncthreads();
    }
    zero_tail(out, covered_bytes<kDimM>(table, s), out_size);
}

// Self-test of the bounded pipeline wait: one thread waits on an mbarrier
// that nothing arrives at; the wait gives up after `limit` clocks and raises
// the timeout flag, exactly as a stalled load would in the kernels above.
__global__ void bounded_wait_selftest(long long limit) {
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_mbar_init();
        if (!mbar_wait_bounded(&bar, 0, limit)) atomicOr(&g_mx_flags, kFlagWaitTimeout);
    }
}

// ------------------------------------------------------------------ host side
constexpr int64_t kMaxExtent = (1ll << 31) - (1ll << 14);
constexpr int kMaxDevices = 128;

struct DeviceInfo {
    bool ready = false;
    int sms = 0;
    int occ_tma[2] = {0, 0};   // [dimM]
    int occ_fallback = 0;
};

// Shared memory of the flat-row kernel for a given row stride and column count.
FlatShape flat_shape(int64_t row_stride, int64_t padded_cols) {
    FlatShape f;
    f.row_stride = (int32_t)row_stride;
    const int64_t span = 16 + kTileRows * row_stride + 256;   // delta, rows, last partial quad
    f.stage_bytes = (int32_t)((span + kFlatBoxBytes - 1) / kFlatBoxBytes * kFlatBoxBytes);
    f.staging_bytes = (int32_t)(((padded_cols / 4) * 512 + 1023) / 1024 * 1024);
    return f;
}

int flat_smem_bytes(const FlatShape &f, int stages, bool direct) {
    return stages * f.stage_bytes + (direct ? 0 : 2 * f.staging_bytes) + 128;
}

// The flat kernel instance for rows of `padded_cols` columns.
bool flat_narrow(int64_t padded_cols) { return padded_cols <= kFlatNarrowCols; }

// The CUDA error behind the calling thread's latest MX_ERR_CUDA.
thread_local cudaError_t t_last_error = cudaSuccess;

mx_status cuda_status(cudaError_t e) {
    if (e == cudaSuccess) return MX_OK;
    t_last_error = e;
    return MX_ERR_CUDA;
}

std::mutex g_mu;
DeviceInfo g_dev[kMaxDevices];
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    std::call_once(g_encode_once, [] {
        void *fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    });
    return g_encode;
}

PFN_cuCtxGetCurrent_v4000 g_ctx_current = nullptr;
std::once_flag g_ctx_once;

PFN_cuCtxGetCurrent_v4000 ctx_current_fn() {
    std::call_once(g_ctx_once, [] {
        void *fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &fn, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            g_ctx_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(fn);
    });
    return g_ctx_current;
}

mx_status device_info(const DeviceInfo **out) {
    int dev = 0;
    if (cudaError_t e = cudaGetDevice(&dev); e != cudaSuccess) return cuda_status(e);
    if (dev < 0 || dev >= kMaxDevices) return MX_ERR_UNSUPPORTED;
    // The tensor-map encoder is a driver call and needs a context current in
    // this thread.  A thread whose first CUDA work is this call has none yet:
    // bind the device's primary context then, and only then, so that a
    // context the caller made current (the primary one or its own) stays.
    auto get_current = ctx_current_fn();
    if (get_current == nullptr) return cuda_status(cudaErrorSymbolNotFound);
    CUcontext cur = nullptr;
    if (CUresult r = get_current(&cur); r != CUDA_SUCCESS) return cuda_status(static_cast<cudaError_t>(r));
    if (cur == nullptr) {
        if (cudaError_t e = cudaSetDevice(dev); e != cudaSuccess) return cuda_status(e);
    }
    std::lock_guard<std::mutex> lock(g_mu);
    DeviceInfo &d = g_dev[dev];
    if (!d.ready) {
        if (cudaError_t e = cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev); e != cudaSuccess)
            return cuda_status(e);
        const int flat_max = flat_smem_bytes(flat_shape(kFlatMaxStride, kFlatMaxStride), kFlatStages, true);
        const FlatShape narrow_max = flat_shape(kFlatMaxStride, kFlatNarrowCols);
        const cudaError_t setup[] = {
            cudaFuncSetAttribute(rearrange_flat_tma<8, kFlatStages, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 flat_max),
            cudaFuncSetAttribute(rearrange_flat_tma<4, 2, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 flat_smem_bytes(narrow_max, 2, true)),
            cudaFuncSetAttribute(rearrange_flat_tma<4, 2, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 flat_smem_bytes(narrow_max, 2, false)),
            cudaFuncSetAttribute(rearrange_tma_m, cudaFuncAttributeMaxDynamicSharedMemorySize, tma_smem_bytes<true>()),
            cudaFuncSetAttribute(rearrange_tma_k, cudaFuncAttributeMaxDynamicSharedMemorySize, tma_smem_bytes<false>()),
            cudaOccupancyMaxActiveBlocksPerMultiprocessor(&d.occ_tma[1], rearrange_tma_m, kThreads,
                                                          tma_smem_bytes<true>()),
            cudaOccupancyMaxActiveBlocksPerMultiprocessor(&d.occ_tma[0], rearrange_tma_k, kThreads,
                                                          tma_smem_bytes<false>()),
            cudaOccupancyMaxActiveBlocksPerMultiprocessor(&d.occ_fallback, rearrange_fallback<true, true>, kThreads, 0),
        };
        for (cudaError_t e : setup)
            if (e != cudaSuccess) return cuda_status(e);
        if (d.occ_tma[0] < 1 || d.occ_tma[1] < 1 || d.occ_fallback < 1) return cuda_status(cudaErrorInvalidConfiguration);
        d.ready = true;
    }
    *out = &d;
    return MX_OK;
}

// A plain stream-ordered launch.  The kernels carry the programmatic
// dependent launch handshake (griddepcontrol), but they are launched without
// programmatic stream serialization: on a B200 it gained nothing between
// launches of the same kernel and cost 1-2 us at every switch from one kernel
// to another (CUDA graphs, cold inputs), and in use a different kernel always
// precedes these.  The launch's own return code reports a failed launch.
template <typename... KArgs, typename... Args>
cudaError_t launch_kernel_block(void (*kernel)(KArgs...), int grid, int block, int smem, cudaStream_t stream,
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

template <typename... KArgs, typename... Args>
cudaError_t launch_kernel(void (*kernel)(KArgs...), int grid, int smem, cudaStream_t stream, Args... args) {
    return launch_kernel_block(kernel, grid, kThreads, smem, stream, args...);
}

int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }
int64_t round_up(int64_t a, int64_t b) { return ceil_div(a, b) * b; }

bool tma_eligible(const void *scales, int64_t rows, int64_t cols, int64_t row_stride) {
    return rows >= 1 && cols >= 1 && (reinterpret_cast<uintptr_t>(scales) & 15u) == 0 &&
           (row_stride & 15) == 0 && row_stride < (1ll << 40);
}

bool word_eligible(const void *scales, int64_t row_stride) {
    return (reinterpret_cast<uintptr_t>(scales) & 3u) == 0 && (row_stride & 3) == 0;
}

bool flat_aligned(const void *scales, int64_t cols, int64_t row_stride) {
    return (reinterpret_cast<uintptr_t>(scales) & 15u) == 0 && (row_stride & 3) == 0 && (cols & 3) == 0;
}

bool flat_eligible(mx_group_dim dim, const void *scales, int64_t rows, int64_t cols, int64_t row_stride) {
    return dim == MX_GROUPS_M && rows >= 1 && cols >= 1 && row_stride <= kFlatMaxStride &&
           flat_aligned(scales, cols, row_stride) && ((rows - 1) * row_stride + cols) / 4 < INT_MAX - (1 << 16);
}

mx_path auto_path(mx_group_dim dim, const void *scales, int64_t rows, int64_t cols, int64_t row_stride) {
    if (rows == 0 || cols == 0) return MX_PATH_WORD;   // nothing to load
    if (tma_eligible(scales, rows, cols, row_stride)) return MX_PATH_TMA;
    if (flat_eligible(dim, scales, rows, cols, row_stride)) return MX_PATH_FLAT;
    if (word_eligible(scales, row_stride)) return MX_PATH_WORD;
    return MX_PATH_BYTE;
}

mx_status run(mx_group_dim dim, const uint8_t *scales, int64_t rows, int64_t cols, int64_t row_stride,
              const int32_t *ends, int32_t G, uint8_t *out, mx_path path, cudaStream_t stream) {
    if (dim != MX_GROUPS_M && dim != MX_GROUPS_K) return MX_ERR_INVALID_ARG;
    if (path < MX_PATH_AUTO || path > MX_PATH_FLAT) return MX_ERR_INVALID_ARG;
    if (G < 1 || G > MX_MAX_GROUPS) return MX_ERR_INVALID_ARG;
    if (rows < 0 || cols < 0 || rows > kMaxExtent || cols > kMaxExtent) return MX_ERR_INVALID_ARG;
    if (row_stride < cols) return MX_ERR_INVALID_ARG;
    if (ends == nullptr) return MX_ERR_INVALID_ARG;
    const bool dim_m = dim == MX_GROUPS_M;
    const size_t size = mx_rearranged_size(dim, rows, cols, G);
    if (size > 0 && out == nullptr) return MX_ERR_INVALID_ARG;
    if (rows > 0 && cols > 0 && scales == nullptr) return MX_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(out) & 15u) != 0) return MX_ERR_MISALIGNED;
    if (size == 0) return MX_OK;

    Shape s;
    s.rows = (int32_t)rows;
    s.cols = (int32_t)cols;
    s.G = G;
    s.padded_cols = (int32_t)round_up(cols, 4);
    s.padded_rows = (int32_t)round_up(rows, 128);
    s.col_chunks = (int32_t)ceil_div(s.padded_cols, kChunkCols);
    // Upper bound on work items, known without reading the offsets.
    const int64_t bound = dim_m ? (ceil_div(rows, 128) + G) * s.col_chunks
                                : ceil_div(rows, 128) * (ceil_div(cols, kChunkCols) + G);
    if (bound > INT_MAX) return MX_ERR_UNSUPPORTED;

    const bool degenerate = rows == 0 || cols == 0;
    if (path == MX_PATH_AUTO) path = auto_path(dim, scales, rows, cols, row_stride);
    if (degenerate) path = MX_PATH_WORD;  // nothing to load: only the zero fill runs
    if (path == MX_PATH_TMA && !tma_eligible(scales, rows, cols, row_stride)) return MX_ERR_MISALIGNED;
    if (path == MX_PATH_FLAT && (!dim_m || row_stride > kFlatMaxStride)) return MX_ERR_UNSUPPORTED;
    if (path == MX_PATH_FLAT && !flat_eligible(dim, scales, rows, cols, row_stride)) return MX_ERR_MISALIGNED;
    if (path == MX_PATH_WORD && !degenerate && !word_eligible(scales, row_stride)) return MX_ERR_MISALIGNED;

    const DeviceInfo *d = nullptr;
    if (mx_status st = device_info(&d); st != MX_OK) return st;
    const int64_t work = bound > 0 ? bound : 1;
    cudaError_t launched = cudaSuccess;

    if (path == MX_PATH_TMA) {
        auto encode = encode_fn();
        if (encode == nullptr) return cuda_status(cudaErrorSymbolNotFound);
        CUtensorMap map;
        cuuint64_t gdim[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
        cuuint64_t gstride[1] = {(cuuint64_t)row_stride};
        cuuint32_t box[2] = {(cuuint32_t)(dim_m ? kPitchSw : kPitchPlain), (cuuint32_t)kTileRows};
        cuuint32_t estride[2] = {1, 1};
        CUresult r = encode(&map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t *>(scales), gdim, gstride,
                            box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE,
                            dim_m ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) return cuda_status(static_cast<cudaError_t>(r));   // driver code
        const int64_t cap = (int64_t)d->sms * d->occ_tma[dim_m ? 1 : 0];
        const int grid = (int)(work < cap ? work : cap);
        launched = dim_m ? launch_kernel(rearrange_tma_m, grid, tma_smem_bytes<true>(), stream, map, ends, out,
                                      (int64_t)size, s)
                         : launch_kernel(rearrange_tma_k, grid, tma_smem_bytes<false>(), stream, map, ends, out,
                                      (int64_t)size, s);
    } else if (path == MX_PATH_FLAT) {
        auto encode = encode_fn();
        if (encode == nullptr) return cuda_status(cudaErrorSymbolNotFound);
        CUtensorMap map;
        cuuint64_t gdim[1] = {(cuuint64_t)(((rows - 1) * row_stride + cols) / 4)};
        cuuint64_t gstride[1] = {0};
        cuuint32_t box[1] = {(cuuint32_t)kFlatBoxWords};
        cuuint32_t estride[1] = {1};
        CUresult r = encode(&map, CU_TENSOR_MAP_DATA_TYPE_UINT32, 1, const_cast<uint8_t *>(scales), gdim, gstride,
                            box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) return cuda_status(static_cast<cudaError_t>(r));   // driver code
        const FlatShape f = flat_shape(row_stride, s.padded_cols);
        const bool narrow = flat_narrow(s.padded_cols);
        const int block = narrow ? 128 : kThreads;
        const int stages = narrow ? 2 : kFlatStages;
        // Direct stores, except for the 4-warp kernel when the items outnumber
        // two waves of the grid (each CTA then streams several items, and the
        // staged bulk stores overlap them better).
        auto kernel = narrow ? rearrange_flat_tma<4, 2, true> : rearrange_flat_tma<8, kFlatStages, true>;
        int smem = flat_smem_bytes(f, stages, true);
        int occ = 0;
        if (cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kernel, block, smem);
            e != cudaSuccess || occ < 1)
            return cuda_status(e != cudaSuccess ? e : cudaErrorInvalidConfiguration);
        if (narrow && work > 2ll * d->sms * occ) {
            kernel = rearrange_flat_tma<4, 2, false>;
            smem = flat_smem_bytes(f, stages, false);
            if (cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kernel, block, smem);
                e != cudaSuccess || occ < 1)
                return cuda_status(e != cudaSuccess ? e : cudaErrorInvalidConfiguration);
        }
        const int64_t cap = (int64_t)d->sms * occ;
        const int grid = (int)(work < cap ? work : cap);
        launched = launch_kernel_block(kernel, grid, block, smem, stream, map, ends, out, (int64_t)size, s, f);
    } else {
        const int64_t cap = (int64_t)d->sms * d->occ_fallback * 4;
        const int grid = (int)(work < cap ? work : cap);
        const bool word = path == MX_PATH_WORD;
        auto kernel = dim_m ? (word ? rearrange_fallback<true, true> : rearrange_fallback<true, false>)
                            : (word ? rearrange_fallback<false, true> : rearrange_fallback<false, false>);
        launched = launch_kernel(kernel, grid, 0, stream, scales, row_stride, ends, out, (int64_t)size, s);
    }
    return cuda_status(launched);
}

}  // namespace mx

// Shared with mx_inverse.cu (C++ linkage, not part of the C ABI).
mx_status mx_record_cuda_error(cudaError_t e) { return mx::cuda_status(e); }
cudaError_t mx_inverse_flags(unsigned int *flags, int clear);   // defined in mx_inverse.cu

// A 2-D uint8 tensor map over `rows` rows of `width` bytes at `row_stride`
// (a multiple of 16) from the 16-byte aligned `base`, boxes of box_w x box_h
// with the given swizzle, for the current device (whose primary context is
// made current in this thread first, as the encoder needs).
mx_status mx_encode_rows_map(CUtensorMap *map, const void *base, int64_t width, int64_t rows, int64_t row_stride,
                             uint32_t box_w, uint32_t box_h, CUtensorMapSwizzle swizzle) {
    const mx::DeviceInfo *d = nullptr;
    if (mx_status st = mx::device_info(&d); st != MX_OK) return st;
    auto encode = mx::encode_fn();
    if (encode == nullptr) return mx::cuda_status(cudaErrorSymbolNotFound);
    cuuint64_t gdim[2] = {(cuuint64_t)width, (cuuint64_t)rows};
    cuuint64_t gstride[1] = {(cuuint64_t)row_stride};
    cuuint32_t box[2] = {box_w, box_h};
    cuuint32_t estride[2] = {1, 1};
    CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(base), gdim, gstride, box, estride,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return mx::cuda_status(static_cast<cudaError_t>(r));   // driver code
    return MX_OK;
}

// ------------------------------------------------------------------ C ABI
extern "C" {

size_t mx_rearranged_size(mx_group_dim dim, int64_t rows, int64_t cols, int32_t num_groups) {
    if ((dim != MX_GROUPS_M && dim != MX_GROUPS_K) || rows < 0 || cols < 0 || num_groups < 1 ||
        num_groups > MX_MAX_GROUPS || rows > mx::kMaxExtent || cols > mx::kMaxExtent)
        return 0;
    if (dim == MX_GROUPS_M) return (size_t)((rows + 128ll * num_groups) * mx::round_up(cols, 4));
    return (size_t)(mx::round_up(rows, 128) * (cols + 4ll * num_groups));
}

mx_status mx_rearrange_m_groups(const uint8_t *scales, int64_t rows, int64_t cols, int64_t row_stride,
                                const int32_t *group_end_offsets, int32_t num_groups, uint8_t *out,
                                cudaStream_t stream) {
    return mx::run(MX_GROUPS_M, scales, rows, cols, row_stride, group_end_offsets, num_groups, out,
                   MX_PATH_AUTO, stream);
}

mx_status mx_rearrange_k_groups(const uint8_t *scales, int64_t rows, int64_t cols, int64_t row_stride,
                                const int32_t *group_end_offsets, int32_t num_groups, uint8_t *out,
                                cudaStream_t stream) {
    return mx::run(MX_GROUPS_K, scales, rows, cols, row_stride, group_end_offsets, num_groups, out,
                   MX_PATH_AUTO, stream);
}

mx_status mx_rearrange_ex(mx_group_dim dim, const uint8_t *scales, int64_t rows, int64_t cols,
                          int64_t row_stride, const int32_t *group_end_offsets, int32_t num_groups,
                          uint8_t *out, mx_path path, cudaStream_t stream) {
    return mx::run(dim, scales, rows, cols, row_stride, group_end_offsets, num_groups, out, path, stream);
}

mx_path mx_select_path(mx_group_dim dim, const void *scales, int64_t rows, int64_t cols, int64_t row_stride) {
    return mx::auto_path(dim, scales, rows, cols, row_stride);
}

const char *mx_status_string(mx_status status) {
    switch (status) {
        case MX_OK: return "ok";
        case MX_ERR_INVALID_ARG: return "invalid argument";
        case MX_ERR_MISALIGNED: return "misaligned pointer or stride for the requested path";
        case MX_ERR_UNSUPPORTED: return "shape beyond the supported index range";
        case MX_ERR_CUDA: return "CUDA call failed";
    }
    return "unknown status";
}

mx_status mx_device_flags(uint32_t *flags, int clear) {
    if (flags == nullptr) return MX_ERR_INVALID_ARG;
    unsigned int v = 0, inv = 0;
    if (cudaError_t e = cudaMemcpyFromSymbol(&v, mx::g_mx_flags, sizeof(v)); e != cudaSuccess)
        return mx::cuda_status(e);
    if (cudaError_t e = mx_inverse_flags(&inv, clear); e != cudaSuccess) return mx::cuda_status(e);
    *flags = v | inv;
    if (clear) {
        const unsigned int zero = 0;
        if (cudaError_t e = cudaMemcpyToSymbol(mx::g_mx_flags, &zero, sizeof(zero)); e != cudaSuccess)
            return mx::cuda_status(e);
    }
    return MX_OK;
}

mx_status mx_selftest_bounded_wait(int64_t limit_cycles, cudaStream_t stream) {
    if (limit_cycles < 1 || limit_cycles > (1ll << 32)) return MX_ERR_INVALID_ARG;
    void *args[] = {&limit_cycles};
    return mx::cuda_status(cudaLaunchKernel(reinterpret_cast<const void *>(mx::bounded_wait_selftest), dim3(1),
                                            dim3(32), args, 0, stream));
}

int mx_last_cuda_error(void) { return (int)mx::t_last_error; }

int mx_version(void) { return 100; }

}  // extern "C"
