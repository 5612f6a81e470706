// fd_split.cuh -- the split stage of decode attention, optionally with the
// final reduction fused in (one thread block per run of key/value tiles; see
// fd_partition.cuh for how runs are cut).
//
// "Flash-Decoding for long-context inference", section "A faster attention
// for decoding: Flash-Decoding": each split computes the attention of the
// query with its chunk of keys/values and writes one extra scalar per row,
// the log-sum-exp; the softmax can be built up tile by tile ("the
// attention/softmax can be calculated iteratively"), which is what the
// running max / running sum below do. A final reduction rescales the splits
// by their log-sum-exps (fd_merge.cuh).
//
// Block layout (352 threads, 384 for paged caches; one block per SM):
//   warp 8      producer: one lane streams K and V tiles (64 tokens x D bf16
//               each) from HBM into a ring of shared-memory stages with 3-D
//               TMA loads, 128-byte swizzled, mbarrier completion; with each
//               group's first tile of a row segment it also bulk-copies that
//               row's query heads into the stage. Paged caches: it brings K
//               and the query heads, and warp 11 (one lane) brings V.
//   warps 0..7  consumers in two groups of four. Group q takes the tiles with
//               sequence number = q (mod 2), so each SM sub-partition runs two
//               independent chains; warp w of a group owns tokens
//               [16w, 16w+16) of its tiles. Per tile: logits, online-softmax
//               update of the running max m and sum l per query head, and
//               the rescaled accumulation of p * v. At the end of a row
//               segment each warp only copies its (m, l, o) into one of two
//               shared-memory merge buffers and goes on.
//   warps 9,10  finishers: merge the eight warps' states of each segment and
//               store the result (whole row) or the segment (workspace), off
//               the consumers' path. Fused form: after storing a segment they
//               take a ticket on its row (atomic counter in the workspace, no
//               waiting); the block that completes a row queues it, and at
//               the end of its run all consumer and finisher threads merge
//               the queued rows' segments and reset their counters. Rows
//               with no tokens are written by block u % P.
// Two consumer forms:
//   * grouped heads (g = Hq/Hkv >= 2): the g query heads that share one kv
//     head form a small dense contraction, run on tensor cores with
//     mma.sync m16n8k16 (bf16 in, fp32 accumulate): S^T[16 tok x 8 heads] =
//     K[16 x D] Q^T and O^T[D x 8 heads] += V^T[D x 16 tok] P^T, P split
//     into a bf16 high part and a bf16 remainder so P V keeps ~16 bits of P.
//     Every K/V byte is read once for the whole group.
//   * one head per kv head (g = 1): CUDA-core dot products, 16 (D=128) or 8
//     (D=64) lanes per token, reduced with warp shuffles.
#pragma once

#include "fd_merge.cuh"
#include "fd_partition.cuh"
#include "fd_ptx.cuh"

namespace fd {

// Consumers: 8 warps in groups that take turns on tiles. By default two
// groups of four warps, 16 tokens of each 64-token tile per warp; a consumer
// type can declare 32 tokens per warp (four groups of two warps).
constexpr int kGroups = 2;                        // default: consumer groups alternating tiles
constexpr int kSliceWarps = 4;                    // default: warps per group (16 tokens each)
constexpr int kConsumerWarps = kGroups * kSliceWarps;
constexpr int kConsumerThreads = kConsumerWarps * 32;
constexpr int kProducerWarp = kConsumerWarps;     // warp 8
constexpr int kFinisherWarps = 2;                 // warps 9, 10
constexpr int kFinisherThreads = kFinisherWarps * 32;
constexpr int kSplitThreads = kConsumerThreads + 32 + kFinisherThreads;
constexpr int kWorkerThreads = kConsumerThreads + kFinisherThreads;   // all but the producer
// Paged caches add a second producer, warp 11, that brings the V boxes while
// warp 8 brings K and the query heads: a TMA copy costs its issuing thread a
// fixed time, which dominates the small boxes of small pages, and copies from
// two warps start in parallel.
constexpr int kVProducerWarp = kProducerWarp + 1 + kFinisherWarps;
template <bool kPaged>
constexpr int split_threads() { return kSplitThreads + (kPaged ? 32 : 0); }
constexpr int kPendingMax = 4;                    // rows or chunks a block completes (a run cuts at most 2
                                                  // rows; each completed chunk may complete its row)
constexpr int kBarFinishers = 1, kBarWorkers = 2; // named barrier ids
constexpr int kPrefetchTiles = 8;                 // tiles guessed into L2 before the dependency wait
constexpr int kWarpTokens = 16;                   // default tokens of a tile owned by one consumer warp
constexpr int kBoxBytes = kTileTokens * 128;      // one TMA box: 64 rows x 128 bytes (64 bf16)
constexpr int kSmemLimit = 232448;                // 227 KiB opt-in shared memory per block
#ifdef FD_DEBUG
constexpr uint64_t kWaitLimitNs = 50000000ull;    // debug builds: a bounded wait gives up after 50 ms
#else
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // a bounded wait gives up after 2 s
#endif



struct SplitParams {
    const uint16_t *q;        // [B, Hq, D]
    const int32_t *seqlens;   // [B]
    float *out;               // [B, Hq, D]
    float *lse;               // [B, Hq]
    float *seg_out;           // [slots, g, D]
    float *seg_lse;           // [slots, g]
    int *row_tickets;         // [B * Hkv], zero between calls (fused form only)
    int *chunk_tickets;       // [slots], one per possible chunk start, zero between calls (fused form only)
    int B, Hq, Hkv, g, Lmax, P;
    int q_len;                // queries per sequence (1: plain decode)
    int cols;                 // g * q_len: (query, head) columns per (sequence, kv head) row
    float scale_log2e;        // scale * log2(e): logits are kept in base 2
    // paged caches only
    const int32_t *block_table;   // [B, max_pages]: page of each sequence's logical page
    int max_pages;            // block-table row length (a multiple of 4)
    int page_shift;           // log2(page_size)
    int kv_nhd;               // 0: pages [num_pages, Hkv, page_size, D]; 1: [num_pages, page_size, Hkv, D]
    int num_pages;            // pages in each pool
    // 8-bit caches only: value of a cached element = scale[kv head] * decode(code)
    const float *k_scale;     // [Hkv]
    const float *v_scale;     // [Hkv]
    // contiguous caches only: the K and V arrays, for the bulk L2 prefetch before the dependency wait
    const void *k_base;
    const void *v_base;
    int debug_withhold;       // debug builds: block 0 issues no copy for this tile (a wait then runs out); -1: off
    int debug_spoil_guess;    // debug builds: make every block's pre-wait guess of its start wrong
};

// Sizes the debug checks compare with.
__device__ __forceinline__ size_t out_rows(const SplitParams &p) {
    return static_cast<size_t>(p.B) * p.q_len * p.Hq;
}
__device__ __forceinline__ size_t seg_rows(const SplitParams &p) {
    return (static_cast<size_t>(p.P) + static_cast<size_t>(p.B) * p.Hkv - 1) * p.cols;
}

constexpr int kPageWindow = 1024;                 // block-table entries staged in shared memory

// One consumer warp's state in a merge buffer: o[G][D] with a row stride of
// D + 4 floats, then m[G], l[G], padded to a multiple of 4 floats. The extra
// 4 floats per head put the accumulator columns that lanes 4 apart hold
// (heads 2c and 2c + 2) 8 banks apart, so a warp's stores of its
// accumulators meet no bank conflict.
template <int D>
__host__ __device__ constexpr int merge_head_stride() { return D + 4; }
template <int D, int G>
__host__ __device__ constexpr int merge_warp_floats() { return (G * merge_head_stride<D>() + 2 * G + 3) / 4 * 4; }

// Byte offset, inside a K or V tile, of 16-byte chunk j (0..7) of the
// 64-element half `half` of token t. Default layout (one TMA box per half):
// [half][64 tokens][128 B]. Interleaved layout (one box covers both halves
// of a token, used for small pages at D = 128): [64 tokens][half][128 B].
// Either way a 128-byte row R keeps the 128-byte swizzle: chunk j sits at
// position j ^ (R & 7).
template <bool kInter>
__device__ __forceinline__ uint32_t tile_offset(int t, int half, int j) {
    if constexpr (kInter) {
        const int R = 2 * t + half;
        return static_cast<uint32_t>(R * 128 + ((j ^ (R & 7)) << 4));
    } else {
        return static_cast<uint32_t>(half * kBoxBytes + t * 128 + ((j ^ (t & 7)) << 4));
    }
}

// Output row of column `col` of row (b, h): column col = j*g + i is query j,
// query head h*g + i; out is [B, q_len, Hq, D] and lse [B, q_len, Hq].
__device__ __forceinline__ size_t out_row(const SplitParams &p, int b, int h, int col) {
    const int j = col / p.g, i = col - j * p.g;
    return (static_cast<size_t>(b) * p.q_len + j) * p.Hq + static_cast<size_t>(h) * p.g + i;
}

// E = bytes per cached element: 2 (bf16) or 1 (8-bit codes).
template <int D, int G, int E = 2, bool kPaged = false>
struct SplitConfig {
    static constexpr int kRowBytes = D * E;                                // one token of one head
    static constexpr int kBoxRowBytes = kRowBytes < 128 ? kRowBytes : 128; // a box row = one swizzle span
    static constexpr int kBoxCols = kBoxRowBytes / E;                      // head-dim elements per box
    static constexpr int kBoxes = D / kBoxCols;                            // boxes per tile
    static constexpr int kBoxBytes = kTileTokens * kBoxRowBytes;
    static constexpr int kTileBytes = kTileTokens * kRowBytes;             // one K (or V) tile
    static constexpr int kQSlotBytes = (G * D * 2 + 1023) / 1024 * 1024;   // query heads of a row (bf16)
    static constexpr int kStageBytes = 2 * kTileBytes + kQSlotBytes;       // multiple of 1024 (swizzle)
    static constexpr int kWarpFloats = merge_warp_floats<D, G>();          // o, m, l of one warp
    static constexpr int kMergeFloats = kConsumerWarps * kWarpFloats;      // one merge buffer
    static constexpr int kCtrlBytes = 2048;                                // barriers, start info, queue, weights
    static constexpr int kPageBytes = kPageWindow * 4;                     // block-table window (paged)
    static constexpr int kFixedBytes = 1024 + kCtrlBytes + (kPaged ? 2 : 1) * kPageBytes;   // one window per producer
    // 128 KiB of K/V tiles in flight (measured best for bf16: 4 stages at
    // D = 128), as many as fit next to one merge buffer, in whole pairs
    static constexpr int fit_stages(int s) {
        return s > 2 && kFixedBytes + s * kStageBytes + kMergeFloats * 4 > kSmemLimit ? fit_stages(s - 2) : s;
    }
    static constexpr int kStages = fit_stages(1024 / kRowBytes);
    static constexpr int kRingBytes = kStages * kStageBytes;
    static constexpr int kMergeBufs = kFixedBytes + kRingBytes + 2 * kMergeFloats * 4 <= kSmemLimit ? 2 : 1;
    static constexpr int kSmemBytes = kFixedBytes + kRingBytes + kMergeBufs * kMergeFloats * 4;
    // Each consumer group owns whole stages: a stage shared by both groups
    // could be waited on two phases ahead of a tile still in flight, where a
    // parity wait would pass on the older phase.
    static_assert(kStages % 2 == 0, "stages come in pairs");
    static_assert(kStageBytes % 1024 == 0, "stages must keep the 1024-byte swizzle alignment");
    static_assert(kSmemBytes <= kSmemLimit, "shared memory over the limit");
};

struct Cursor {
    int b, h, tile, n;        // row (b, h), tile index inside the row, tiles of sequence b
    long long first;          // flat index of the row's first tile
};

struct PendingRow {
    int b, h;                 // the row
    int chunk;                // -1: the row is complete; c >= 0: chunk c of a two-level row is
    RowRuns rr;               // the runs holding the row's tiles
};

struct StartInfo {
    long long count;          // tiles in this block's run
    long long N;              // tiles in the whole batch
    long long first;          // flat index of the start row's first tile
    int b, h, tile, n;
    int abort;                // set when a bounded wait gave up
    int restart;              // the producer's guessed first tiles were wrong: the ring restarts one phase on
    int last_buf;             // merge buffer holding the run's last segment
    int npending;             // rows this block completed (fused form)
    PendingRow pending[kPendingMax];
    RowRuns last_rr;          // the runs of the run's last segment's row (worked out ahead of its ticket)
};

// Bounded mbarrier wait. Returns false if the block is aborting or the limit
// passes (then it marks the abort and the device error word).
__device__ __forceinline__ bool wait_bounded(uint64_t *bar, uint32_t parity, volatile int *abort) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort) return false;
    const uint64_t t0 = global_timer_ns();
    while (true) {
        if (mbar_try_wait(bar, parity)) return true;
        if (*abort) return false;
        if (global_timer_ns() - t0 > kWaitLimitNs) {
            *abort = 1;
            atomicExch(&g_fd_error_word, -10 /* FD_ERR_TIMEOUT */);
            return false;
        }
    }
}

// Wait for warp 0 to publish the block's real start (phase 0 of `bar`). If
// the bounded wait gives up, the device error word is set; the block then
// goes on with whatever the start record holds and the call is reported as
// failed by fd_device_status.
__device__ __forceinline__ void wait_start(uint64_t *bar) {
    if (mbar_try_wait(bar, 0)) return;
    const uint64_t t0 = global_timer_ns();
    while (!mbar_try_wait(bar, 0))
        if (global_timer_ns() - t0 > kWaitLimitNs) {
            atomicExch(&g_fd_error_word, -10 /* FD_ERR_TIMEOUT */);
            return;
        }
}

// After a wait gave up: wait once more, bounded and regardless of the abort
// flag, for a phase whose copies were issued, so that no copy still lands in
// this block's shared memory after it exits.
__device__ __forceinline__ void drain_phase(uint64_t *bar, uint32_t parity) {
    const uint64_t t0 = global_timer_ns();
    while (!mbar_try_wait(bar, parity))
        if (global_timer_ns() - t0 > kWaitLimitNs) return;
}

// The producer's copies still possibly in flight when it gives up: the last
// load issued into each stage (`issued` tiles so far, stage = tile % stages)
// and the block-table window (when `window_pending`).
template <int kStages>
__device__ __forceinline__ void drain_copies(uint64_t *full, uint32_t issued, uint64_t *pbar, bool window_pending,
                                             uint32_t win_phase) {
    for (uint32_t s = 0; s < static_cast<uint32_t>(kStages) && s < issued; ++s) {
        const uint32_t n = (issued - 1 - s) / kStages + 1;   // loads issued into stage s
        drain_phase(&full[s], (n - 1) & 1u);
    }
    if (window_pending) drain_phase(pbar, win_phase);
}

// Contiguous caches: ask L2 for tiles [t0, t1) of row z of K and of V, as
// one bulk prefetch each (clipped to the row's Lmax tokens; nothing past the
// row is touched).
template <int kRowBytes>
__device__ __forceinline__ void prefetch_row_span(const SplitParams &p, int z, int t0, int t1) {
    const int tok0 = t0 * kTileTokens, tok1 = min(t1 * kTileTokens, p.Lmax);
    if (tok1 <= tok0) return;
    const size_t off = (static_cast<size_t>(z) * p.Lmax + tok0) * kRowBytes;
    const uint32_t bytes = static_cast<uint32_t>(tok1 - tok0) * kRowBytes;
    bulk_prefetch_l2(static_cast<const uint8_t *>(p.k_base) + off, bytes);
    bulk_prefetch_l2(static_cast<const uint8_t *>(p.v_base) + off, bytes);
}

__device__ __forceinline__ int row_tiles(const int32_t *seqlens, int b, int Lmax) {
    return tiles_of(clamp_len(__ldg(seqlens + b), Lmax));
}

// L2-only read (no L1 line kept): for a guess made before the previous grid
// has finished, which must not leave a stale copy behind for the real read.
__device__ __forceinline__ int row_tiles_l2(const int32_t *seqlens, int b, int Lmax) {
    return tiles_of(clamp_len(__ldcg(seqlens + b), Lmax));
}

template <bool kL2Only>
__device__ __forceinline__ int tiles_at(const int32_t *seqlens, int b, int Lmax) {
    return kL2Only ? row_tiles_l2(seqlens, b, Lmax) : row_tiles(seqlens, b, Lmax);
}

// One K and one V tile of a contiguous cache (tokens y .. y+63 of row z)
// into the stage. Default layout: one 3-D box per 64 head-dim elements.
// Interleaved layout (bf16, D = 128): one 4-D box {64 elements, 2 halves,
// 64 tokens, 1 row} per tile, [token][half][128 B] in shared memory, so the
// producer issues two copies per tile instead of four (every copy costs its
// issuing thread a fixed time, taken from the warps sharing its scheduler).
template <class Cfg, bool kInter>
__device__ __forceinline__ void load_tile(uint8_t *kt, uint8_t *vt, const CUtensorMap *tm_k, const CUtensorMap *tm_v,
                                          uint64_t *bar, int y, int z, uint64_t policy) {
    if constexpr (kInter) {
        tma_load_4d(kt, tm_k, bar, 0, 0, y, z, policy);
        tma_load_4d(vt, tm_v, bar, 0, 0, y, z, policy);
    } else {
#pragma unroll
        for (int bx = 0; bx < Cfg::kBoxes; ++bx) {
            tma_load_3d(kt + bx * Cfg::kBoxBytes, tm_k, bar, Cfg::kBoxCols * bx, y, z, policy);
            tma_load_3d(vt + bx * Cfg::kBoxBytes, tm_v, bar, Cfg::kBoxCols * bx, y, z, policy);
        }
    }
}

// Next row with at least one tile (only called while tiles remain).
__device__ __forceinline__ void next_row(Cursor &c, const SplitParams &p) {
    c.first += c.n;
    c.tile = 0;
    if (++c.h == p.Hkv) {
        c.h = 0;
        do {
            ++c.b;
            c.n = row_tiles(p.seqlens, c.b, p.Lmax);
        } while (c.n == 0);
    }
}

// Warp 0: total tile count and this block's starting row / tile.
template <bool kGuess>
__device__ __forceinline__ void find_start(const SplitParams &p, StartInfo *info) {
    const int lane = threadIdx.x & 31;
    // the first 32 sequences are read once and kept for the second pass
    const int n_first = lane < p.B ? tiles_at<kGuess>(p.seqlens, lane, p.Lmax) : 0;
    long long total = 0;
    for (int base = 0; base < p.B; base += 32) {
        int n = base == 0 ? n_first : (base + lane < p.B ? tiles_at<kGuess>(p.seqlens, base + lane, p.Lmax) : 0);
        for (int s = 16; s > 0; s >>= 1) n += __shfl_xor_sync(0xffffffffu, n, s);
        total += n;
    }
    const long long N = total * p.Hkv;
    const long long t0 = run_begin(blockIdx.x, N, p.P);
    const long long t1 = run_begin(blockIdx.x + 1, N, p.P);
    int b = 0, h = 0, tile = 0, n = 0;
    long long first = 0;
    if (t1 > t0) {
        long long before = 0;   // Hkv * (tiles of sequences before this chunk)
        for (int base = 0; base < p.B; base += 32) {
            const int nb = base == 0 ? n_first : (base + lane < p.B ? tiles_at<kGuess>(p.seqlens, base + lane, p.Lmax) : 0);
            int incl = nb;
            for (int s = 1; s < 32; s <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, incl, s);
                if (lane >= s) incl += y;
            }
            const long long after = before + static_cast<long long>(p.Hkv) * incl;
            const unsigned hit = __ballot_sync(0xffffffffu, base + lane < p.B && after > t0);
            if (hit) {
                const int src = __ffs(hit) - 1;
                b = base + src;
                n = __shfl_sync(0xffffffffu, nb, src);
                const long long seq0 = __shfl_sync(0xffffffffu, after, src) - static_cast<long long>(p.Hkv) * n;
                const long long off = t0 - seq0;
                h = static_cast<int>(off / n);
                tile = static_cast<int>(off % n);
                first = seq0 + static_cast<long long>(h) * n;
                break;
            }
            before += static_cast<long long>(p.Hkv) * __shfl_sync(0xffffffffu, incl, 31);
        }
    }
    if (lane == 0) {
        info->restart = 0;
        info->count = t1 - t0;
        info->N = N;
        info->first = first;
        info->b = b;
        info->h = h;
        info->tile = tile;
        info->n = n;
        info->abort = 0;
        info->last_buf = 0;
        info->npending = 0;
    }
}

// What the end of a run merges, one entry per queued row or chunk, worked
// out when it is queued (from runs worked out ahead: the partition
// arithmetic divides 64-bit integers, too slow for the end of the run).
enum EndMode : int { kEndChunk = 0, kEndDirect = 1, kEndStaged = 2, kEndFromL2 = 3 };
constexpr int kDirectUnits = 8;   // units read straight from L2 (one round trip)
struct EndPlan {
    Units m[kPendingMax];      // the units the entry folds
    int mode[kPendingMax];     // EndMode
};

// Queue a completed row (chunk = -1) or chunk, with its plan. `stage_floats`:
// the floats of shared memory free at the end of the run.
template <int D>
__device__ __forceinline__ void queue_pending(const SplitParams &p, StartInfo *info, EndPlan *plan, int b, int h,
                                              int chunk, const RowRuns &rr, long long stage_floats) {
    if (!FD_DCHECK(info->npending < kPendingMax)) return;
    const int k = info->npending++;
    info->pending[k] = PendingRow{b, h, chunk, rr};
    const long long u = static_cast<long long>(b) * p.Hkv + h;
    if (chunk >= 0) {
        plan->m[k] = chunk_units(rr, u, chunk);
        plan->mode[k] = kEndChunk;
    } else {
        const Units m = final_units(rr, u, p.cols, D);
        plan->m[k] = m;
        plan->mode[k] = m.count <= kDirectUnits                                    ? kEndDirect
                        : staged_floats(m.count, p.cols, D) <= stage_floats ? kEndStaged
                                                                             : kEndFromL2;
    }
}

// ------------------------------------------------------------------ tickets --
// Called by one thread once the block's segment of row c (runs rr) is stored
// and ordered before this call by a block barrier: take the segment's
// ticket, on the row or, for a two-level row, on the segment's chunk (the
// block's run is blockIdx.x). The acquire-release add makes the stores
// visible at device scope before the count moves, and orders the completing
// block's reads of the other segments after it. A ticket that completes its
// row or chunk queues it; nothing ever waits.
template <int D>
__device__ __forceinline__ void take_ticket(const SplitParams &p, StartInfo *info, EndPlan *plan, const Cursor &c,
                                            const RowRuns &rr, long long N, long long stage_floats) {
    const long long u = static_cast<long long>(c.b) * p.Hkv + c.h;
    int *counter, need, chunk = -1;
    if (!is_two_level(rr, p.cols, D)) {
        if (!FD_DCHECK(u < static_cast<long long>(p.B) * p.Hkv)) return;
        counter = p.row_tickets + u;
        need = rr.count;
    } else {
        chunk = (static_cast<int>(blockIdx.x) - rr.i0) / kFanIn;
        const size_t slot = static_cast<size_t>(rr.i0) + static_cast<size_t>(chunk) * kFanIn + static_cast<size_t>(u);
        if (!FD_DCHECK(chunk >= 0 && chunk < num_chunks(rr) && (slot + 1) * p.cols <= seg_rows(p))) return;
        counter = p.chunk_tickets + slot;
        need = chunk_count(rr, chunk, N, p.P);
    }
    const int prev = atom_add_acq_rel_gpu(counter, 1);
    if (prev == need - 1) queue_pending<D>(p, info, plan, c.b, c.h, chunk, rr, stage_floats);
}

// ------------------------------------------------------------ merge + store --
// Per-warp partial results in shared memory: o[G][D], then m[G], l[G] (m in
// base-2 units). `nthreads` threads (barrier `bar`) merge the eight warps:
// first one thread per head turns the warps' (m, l) into normalised weights
// w[head][warp] = 2^(m_w - M) / sum_w' 2^(m_w' - M) l_w' and the log-sum-exp,
// then every output is sum_w w[head][w] * o_w.
template <int D, int G, class Bar>
__device__ __forceinline__ void merge_warps_and_store(const float *merge, float *weights, const SplitParams &p,
                                                      const Cursor &c, bool whole, size_t slot, int tid,
                                                      int nthreads, Bar bar) {
    constexpr int kWarpFloats = merge_warp_floats<D, G>();
    constexpr int S = merge_head_stride<D>();
    float *lse_h = weights + G * kConsumerWarps;   // [G] natural-log lse per head
    for (int head = tid; head < p.cols; head += nthreads) {
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kConsumerWarps; ++w) M = fmaxf(M, merge[w * kWarpFloats + G * S + head]);
        if (M == -INFINITY) {
#pragma unroll
            for (int w = 0; w < kConsumerWarps; ++w) weights[head * kConsumerWarps + w] = 0.f;
            lse_h[head] = -INFINITY;
        } else {
            float e[kConsumerWarps], lsum = 0.f;
#pragma unroll
            for (int w = 0; w < kConsumerWarps; ++w) {
                e[w] = ex2(merge[w * kWarpFloats + G * S + head] - M);
                lsum = fmaf(e[w], merge[w * kWarpFloats + G * S + G + head], lsum);
            }
            const float inv = 1.f / lsum;
#pragma unroll
            for (int w = 0; w < kConsumerWarps; ++w) weights[head * kConsumerWarps + w] = e[w] * inv;
            lse_h[head] = (M + lg2(lsum)) * kLn2F;
        }
    }
    bar();
    for (int idx = tid; idx < p.cols * D; idx += nthreads) {
        const int head = idx / D, d = idx - head * D;
        float o = 0.f;
#pragma unroll
        for (int w = 0; w < kConsumerWarps; ++w)
            o = fmaf(weights[head * kConsumerWarps + w], merge[w * kWarpFloats + head * S + d], o);
        if (whole) {
            const size_t row = out_row(p, c.b, c.h, head);
            if (!FD_DCHECK(row < out_rows(p))) continue;
            p.out[row * D + d] = o;
            if (d == 0) p.lse[row] = lse_h[head];
        } else {
            const size_t row = slot * p.cols + head;
            if (!FD_DCHECK(row < seg_rows(p))) continue;
            p.seg_out[row * D + d] = o;
            if (d == 0) p.seg_lse[row] = lse_h[head];
        }
    }
}

// ------------------------------------------------- grouped-head consumer --
template <int D, int NT, bool kInter = false>
struct GroupConsumer {
    static constexpr int KS = D / 16;   // k-steps of the logit contraction
    static constexpr int MT = D / 16;   // m-tiles of the P V contraction
    static constexpr int G = 8 * NT;    // heads held (padded)
    static constexpr int kElemBytes = 2;
    static constexpr int kWarpTokens = 16;
    static constexpr bool kInterleaved = kInter;

    uint32_t qf[NT][KS][2];             // Q^T as the B operand, per n-tile
    float m[NT][2], l[NT][2];           // running max (base 2) / partial sum for heads 2c, 2c+1
    float o[NT][MT][4];                 // O^T accumulators
    int shift[NT][2];                   // causal offset of columns 2c, 2c+1: q_len - 1 - query index

    __device__ __forceinline__ void init(const SplitParams &p) {
        const int cc = (threadIdx.x & 31) & 3;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int col = nt * 8 + 2 * cc + e;
                shift[nt][e] = col < p.cols ? p.q_len - 1 - col / p.g : 0;
            }
    }

    __device__ __forceinline__ void set_row(const SplitParams &, int) {}   // bf16 cache: no per-head scales

    __device__ __forceinline__ void reset() {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            m[nt][0] = m[nt][1] = -INFINITY;
            l[nt][0] = l[nt][1] = 0.f;
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) o[nt][mt][0] = o[nt][mt][1] = o[nt][mt][2] = o[nt][mt][3] = 0.f;
        }
    }

    // Q^T fragments from the stage's copy of the row's g query heads ([g][D] bf16).
    __device__ __forceinline__ void load_q(const uint8_t *qs, int g) {
        const int lane = threadIdx.x & 31;
        const int r0 = lane >> 2, cc = lane & 3;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const int head = nt * 8 + r0;
            const bool ok = head < g;
            const uint32_t *qrow = reinterpret_cast<const uint32_t *>(qs + (ok ? head : 0) * D * 2);
#pragma unroll
            for (int ks = 0; ks < KS; ++ks) {
                qf[nt][ks][0] = ok ? qrow[8 * ks + cc] : 0u;
                qf[nt][ks][1] = ok ? qrow[8 * ks + cc + 4] : 0u;
            }
        }
    }

    static __device__ __forceinline__ uint32_t keep_tokens(uint32_t w, int t, int valid) {
        return w & ((t < valid ? 0x0000ffffu : 0u) | (t + 1 < valid ? 0xffff0000u : 0u));
    }

    // One tile: `slice` = this warp's 16-token slice, `valid` = how many of
    // those 16 tokens are inside the row.
    __device__ __forceinline__ void tile(uint32_t k_smem, uint32_t v_smem, int slice, int valid,
                                         float scale_log2e) {
        const int lane = threadIdx.x & 31;
        const int mi = lane >> 3, rr = lane & 7;
        const int r0 = lane >> 2, cc = lane & 3;

        // S^T = K Q^T over this warp's 16 tokens (two accumulators: even and
        // odd k-steps, to halve the dependent mma chain)
        float s[NT][4], s2[NT][4];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) s[nt][e] = s2[nt][e] = 0.f;
        const int krow = kWarpTokens * slice + rr + 8 * (mi & 1);
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) {
            const int d = 16 * ks + 8 * (mi >> 1);
            const uint32_t addr = k_smem + tile_offset<kInter>(krow, d >> 6, (d & 63) >> 3);
            uint32_t a0, a1, a2, a3;
            ldsm_x4(addr, a0, a1, a2, a3);
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                if (ks & 1)
                    mma_bf16_16816(s2[nt], a0, a1, a2, a3, qf[nt][ks][0], qf[nt][ks][1]);
                else
                    mma_bf16_16816(s[nt], a0, a1, a2, a3, qf[nt][ks][0], qf[nt][ks][1]);
            }
        }

        // online softmax per head column; P^T fragments (high + remainder)
        uint32_t bh[NT][2], bl[NT][2];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            float x0 = (s[nt][0] + s2[nt][0]) * scale_log2e, x1 = (s[nt][1] + s2[nt][1]) * scale_log2e;
            float x2 = (s[nt][2] + s2[nt][2]) * scale_log2e, x3 = (s[nt][3] + s2[nt][3]) * scale_log2e;
            // token r of this warp's slice is inside column e's causal range when r < valid - shift
            const int va = valid - shift[nt][0], vb = valid - shift[nt][1];
            if (r0 >= va) x0 = -INFINITY;
            if (r0 >= vb) x1 = -INFINITY;
            if (r0 + 8 >= va) x2 = -INFINITY;
            if (r0 + 8 >= vb) x3 = -INFINITY;
            float ma = fmaxf(x0, x2), mb = fmaxf(x1, x3);
#pragma unroll
            for (int sh = 4; sh < 32; sh <<= 1) {
                ma = fmaxf(ma, __shfl_xor_sync(0xffffffffu, ma, sh));
                mb = fmaxf(mb, __shfl_xor_sync(0xffffffffu, mb, sh));
            }
            const float na = fmaxf(m[nt][0], ma), nb = fmaxf(m[nt][1], mb);
            const float ua = na == -INFINITY ? 0.f : na, ub = nb == -INFINITY ? 0.f : nb;
            const float alpha_a = ex2(m[nt][0] - ua), alpha_b = ex2(m[nt][1] - ub);
            const float p0 = ex2(x0 - ua), p2 = ex2(x2 - ua), p1 = ex2(x1 - ub), p3 = ex2(x3 - ub);
            l[nt][0] = fmaf(l[nt][0], alpha_a, p0 + p2);
            l[nt][1] = fmaf(l[nt][1], alpha_b, p1 + p3);
            m[nt][0] = na;
            m[nt][1] = nb;
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) {
                o[nt][mt][0] *= alpha_a;
                o[nt][mt][2] *= alpha_a;
                o[nt][mt][1] *= alpha_b;
                o[nt][mt][3] *= alpha_b;
            }
            const uint32_t h01 = pack_bf16x2(p0, p1), h23 = pack_bf16x2(p2, p3);
            const uint32_t l01 = pack_bf16x2(p0 - bf16lo_to_f32(h01), p1 - bf16hi_to_f32(h01));
            const uint32_t l23 = pack_bf16x2(p2 - bf16lo_to_f32(h23), p3 - bf16hi_to_f32(h23));
            bh[nt][0] = movmatrix_trans(h01);
            bh[nt][1] = movmatrix_trans(h23);
            bl[nt][0] = movmatrix_trans(l01);
            bl[nt][1] = movmatrix_trans(l23);
        }

        // O^T += V^T P^T
        const int vrow = kWarpTokens * slice + 8 * (mi >> 1) + rr;
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
            const int d = 16 * mt + 8 * (mi & 1);
            const uint32_t addr = v_smem + tile_offset<kInter>(vrow, d >> 6, (d & 63) >> 3);
            uint32_t a0, a1, a2, a3;
            ldsm_x4_trans(addr, a0, a1, a2, a3);
            if (valid < kWarpTokens) {   // rows past the end may hold anything (NaN): zero them
                a0 = keep_tokens(a0, 2 * cc, valid);
                a1 = keep_tokens(a1, 2 * cc, valid);
                a2 = keep_tokens(a2, 8 + 2 * cc, valid);
                a3 = keep_tokens(a3, 8 + 2 * cc, valid);
            }
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                mma_bf16_16816(o[nt][mt], a0, a1, a2, a3, bh[nt][0], bh[nt][1]);
                mma_bf16_16816(o[nt][mt], a0, a1, a2, a3, bl[nt][0], bl[nt][1]);
            }
        }
    }

    __device__ __forceinline__ void to_smem(float *wb) {
        constexpr int S = merge_head_stride<D>();
        const int lane = threadIdx.x & 31;
        const int r0 = lane >> 2, cc = lane & 3;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
            for (int e = 0; e < 2; ++e)
#pragma unroll
                for (int sh = 4; sh < 32; sh <<= 1) l[nt][e] += __shfl_xor_sync(0xffffffffu, l[nt][e], sh);
            const int ha = nt * 8 + 2 * cc, hb = ha + 1;
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) {
                const int d0 = 16 * mt + r0, d1 = d0 + 8;
                wb[ha * S + d0] = o[nt][mt][0];
                wb[hb * S + d0] = o[nt][mt][1];
                wb[ha * S + d1] = o[nt][mt][2];
                wb[hb * S + d1] = o[nt][mt][3];
            }
            if (r0 == 0) {
                wb[G * S + ha] = m[nt][0];
                wb[G * S + hb] = m[nt][1];
                wb[G * S + G + ha] = l[nt][0];
                wb[G * S + G + hb] = l[nt][1];
            }
        }
    }
};

// ------------------------------------------------ one-head (MHA) consumer --
// kTok tokens of each tile per warp: 16 (four warps per group, two groups) or
// 32 (two warps per group, four groups), the 32 as two 16-token halves whose
// dependency chains interleave and which share one rescale of the state.
template <int D, bool kInter = false, int kTok = 16>
struct HeadConsumer {
    static constexpr int G = 1;
    static constexpr int kElemBytes = 2;
    static constexpr int kWarpTokens = kTok;
    static constexpr bool kInterleaved = kInter;
    static constexpr int LPT = D / 8;          // lanes per token (16 bytes = 8 bf16 each)
    static constexpr int TPI = 32 / LPT;       // tokens per warp-wide load
    static constexpr int ITER = 16 / TPI;      // warp-wide loads per 16-token half
    static constexpr int NSUB = kTok / 16;     // 16-token halves
    static_assert(kTok == 16 || kTok == 32, "16 or 32 tokens per warp");

    uint4 qw;                                  // q[d0 .. d0+7] of this lane's 16-byte chunk (bf16 pairs)
    float m, l;                                // running max (base 2, warp-uniform) / lane partial sum
    float acc[8];                              // sum of p * v over this lane's tokens, chunk d0..d0+7

    __device__ __forceinline__ void init(const SplitParams &) {}   // one query, one head: no offsets
    __device__ __forceinline__ void set_row(const SplitParams &, int) {}

    __device__ __forceinline__ void reset() {
        m = -INFINITY;
        l = 0.f;
#pragma unroll
        for (int k = 0; k < 8; ++k) acc[k] = 0.f;
    }

    // q[d0 .. d0+7] from the stage's copy of the row's query head ([D] bf16).
    __device__ __forceinline__ void load_q(const uint8_t *qs, int) {
        const int lane = threadIdx.x & 31;
        const int d0 = 8 * (lane % LPT);
        qw = *reinterpret_cast<const uint4 *>(qs + d0 * 2);
    }

    static __device__ __forceinline__ uint4 lds128(uint32_t addr) {
        uint4 r;
        asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                     : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                     : "r"(addr)
                     : "memory");
        return r;
    }

    __device__ __forceinline__ void tile(uint32_t k_smem, uint32_t v_smem, int slice, int valid,
                                         float scale_log2e) {
        const int lane = threadIdx.x & 31;
        const int half = lane / LPT, chunk = lane % LPT;
        const int d0 = 8 * chunk;
        const int dhalf = d0 >> 6, j = (d0 & 63) >> 3;   // 64-element half of the head dims, chunk in it

        // partial dots over this lane's 8 dims for tokens 16*s + TPI*it + half
        float pd[NSUB][ITER];
#pragma unroll
        for (int s = 0; s < NSUB; ++s)
#pragma unroll
            for (int it = 0; it < ITER; ++it) {
                const int r = kWarpTokens * slice + 16 * s + TPI * it + half;
                const uint4 w = lds128(k_smem + tile_offset<kInter>(r, dhalf, j));
                // q . k over the 8 dims in order, products exact, fp32 sums (-0 start: the
                // first step is the exact product, as a multiply would give)
                float a = fma2_bf16(qw.x, w.x, -0.f);
                a = fma2_bf16(qw.y, w.y, a);
                a = fma2_bf16(qw.z, w.z, a);
                a = fma2_bf16(qw.w, w.w, a);
                pd[s][it] = a;
            }
        // reduce across the LPT lanes of each token while spreading tokens
        // over lanes: after the halving steps lane keeps token index
        // (lane % LPT) / 2 of each half; the last step leaves the full dot in
        // both lanes of each pair.
#pragma unroll
        for (int n = ITER; n > 1; n >>= 1) {
            const bool up = (lane & n) != 0;
#pragma unroll
            for (int k = 0; k < n / 2; ++k)
#pragma unroll
                for (int s = 0; s < NSUB; ++s) {
                    const float send = up ? pd[s][k] : pd[s][k + n / 2];
                    const float keep = up ? pd[s][k + n / 2] : pd[s][k];
                    pd[s][k] = keep + __shfl_xor_sync(0xffffffffu, send, n);
                }
        }
        const int my_it = chunk >> 1;
        float x[NSUB];
        float mx = -INFINITY;   // both lanes of a pair hold the same value: skip the xor-1 step below
#pragma unroll
        for (int s = 0; s < NSUB; ++s) {
            x[s] = (pd[s][0] + __shfl_xor_sync(0xffffffffu, pd[s][0], 1)) * scale_log2e;
            if (16 * s + TPI * my_it + half >= valid) x[s] = -INFINITY;
            mx = fmaxf(mx, x[s]);
        }
#pragma unroll
        for (int sh = 2; sh < 32; sh <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, sh));
        const float mn = fmaxf(m, mx);
        const float mu = mn == -INFINITY ? 0.f : mn;
        const float alpha = ex2(m - mu);
        float pv[NSUB], psum = 0.f;
#pragma unroll
        for (int s = 0; s < NSUB; ++s) {
            pv[s] = ex2(x[s] - mu);
            psum += pv[s];
        }
        l = fmaf(l, alpha, (lane & 1) ? 0.f : psum);
        m = mn;
#pragma unroll
        for (int k = 0; k < 8; ++k) acc[k] *= alpha;

        if (16 * NSUB <= valid) {
            // every token of the warp's slice is inside the row: no per-token
            // test, so all weights and value rows are fetched before the first
            // multiply-add (a test per token keeps each load behind the last)
            float pt[NSUB][ITER];
            uint4 vw[NSUB][ITER];
#pragma unroll
            for (int s = 0; s < NSUB; ++s)
#pragma unroll
                for (int it = 0; it < ITER; ++it) {
                    pt[s][it] = __shfl_sync(0xffffffffu, pv[s], half * LPT + 2 * it);
                    vw[s][it] = lds128(v_smem + tile_offset<kInter>(kWarpTokens * slice + 16 * s + TPI * it + half,
                                                                     dhalf, j));
                }
#pragma unroll
            for (int s = 0; s < NSUB; ++s)
#pragma unroll
                for (int it = 0; it < ITER; ++it) {
                    fma_f32x2_bf16(acc[0], acc[1], pt[s][it], vw[s][it].x);
                    fma_f32x2_bf16(acc[2], acc[3], pt[s][it], vw[s][it].y);
                    fma_f32x2_bf16(acc[4], acc[5], pt[s][it], vw[s][it].z);
                    fma_f32x2_bf16(acc[6], acc[7], pt[s][it], vw[s][it].w);
                }
            return;
        }
        // the row ends inside the slice: rows past it may hold anything (NaN) and are skipped
#pragma unroll
        for (int s = 0; s < NSUB; ++s)
#pragma unroll
            for (int it = 0; it < ITER; ++it) {
                const float pt = __shfl_sync(0xffffffffu, pv[s], half * LPT + 2 * it);
                const int t = 16 * s + TPI * it + half;
                if (t < valid) {
                    const int r = kWarpTokens * slice + t;
                    const uint4 w = lds128(v_smem + tile_offset<kInter>(r, dhalf, j));
                    fma_f32x2_bf16(acc[0], acc[1], pt, w.x);
                    fma_f32x2_bf16(acc[2], acc[3], pt, w.y);
                    fma_f32x2_bf16(acc[4], acc[5], pt, w.z);
                    fma_f32x2_bf16(acc[6], acc[7], pt, w.w);
                }
            }
    }

    __device__ __forceinline__ void to_smem(float *wb) {
        const int lane = threadIdx.x & 31;
#pragma unroll
        for (int s = LPT; s < 32; s <<= 1)
#pragma unroll
            for (int k = 0; k < 8; ++k) acc[k] += __shfl_xor_sync(0xffffffffu, acc[k], s);
        float ls = l;
#pragma unroll
        for (int s = 1; s < 32; s <<= 1) ls += __shfl_xor_sync(0xffffffffu, ls, s);
        if (lane < LPT) {   // two 16-byte stores per lane (the warp's slot is 16-byte aligned)
            reinterpret_cast<float4 *>(wb)[2 * lane] = make_float4(acc[0], acc[1], acc[2], acc[3]);
            reinterpret_cast<float4 *>(wb)[2 * lane + 1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
        }
        if (lane == 0) {
            wb[merge_head_stride<D>()] = m;
            wb[merge_head_stride<D>() + 1] = ls;
        }
    }
};

// ------------------------------------------------------------------ kernel --
template <int D, class Consumer, bool kFused, bool kPaged = false>
__global__ void __launch_bounds__(split_threads<kPaged>(), 1)
    fd_split_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                    const __grid_constant__ CUtensorMap tm_kr, const __grid_constant__ CUtensorMap tm_vr,
                    const SplitParams p) {
    constexpr int G = Consumer::G;
    using Cfg = SplitConfig<D, G, Consumer::kElemBytes, kPaged>;
    constexpr int kTok = Consumer::kWarpTokens;          // tokens per consumer warp and tile
    constexpr int kSlices = kTileTokens / kTok;           // warps per consumer group
    constexpr int kGroupsC = kConsumerWarps / kSlices;    // groups taking turns on tiles
    // Each consumer group owns whole stages: a stage shared by two groups could
    // be waited on two phases ahead of a tile still in flight, where a parity
    // wait would pass on the older phase.
    static_assert(Cfg::kStages % kGroupsC == 0, "each consumer group must own whole stages");
    constexpr int kStages = Cfg::kStages;
    constexpr int kBufs = Cfg::kMergeBufs;

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *ring = smem;                                                  // stages: K tile | V tile | q slot
    float *merge = reinterpret_cast<float *>(ring + Cfg::kRingBytes);      // kBufs x [8 warps][o, m, l]
    uint64_t *full = reinterpret_cast<uint64_t *>(merge + kBufs * Cfg::kMergeFloats);
    uint64_t *empty = full + kStages;
    uint64_t *mfull = empty + kStages;                                     // merge buffer filled (8 warps)
    uint64_t *mempty = mfull + kBufs;                                      // merge buffer drained (finishers)
    uint64_t *pbar = mempty + kBufs;                                       // block-table windows landed (K, V)
    uint64_t *startbar = pbar + 2;                                         // warp 0 has worked out the real start
    StartInfo *info = reinterpret_cast<StartInfo *>(startbar + 1);
    StartInfo *guess = info + 1;                                           // the start as guessed before the wait
    float *weights = reinterpret_cast<float *>(guess + 1);                 // [G][8] merge weights, [G] lse
    constexpr int kWeightFloats = (G * kConsumerWarps + G + 3) / 4 * 4;
    // shared memory free at the end of the run (the ring and merge buffers), in floats
    constexpr long long kStageFloats = (static_cast<long long>(Cfg::kRingBytes) + kBufs * Cfg::kMergeFloats * 4) / 4;
    // a row reduced in one level always fits it
    static_assert(kStageFloats >= (G == 1 ? kTwoLevelSegs * (D + 1) + 4 : kStageBudgetFloats),
                  "a one-level row must fit the shared memory free at the end of the run");
    EndPlan *plan = reinterpret_cast<EndPlan *>(weights + kWeightFloats);  // what the end of the run merges
    static_assert((2 * kStages + 2 * kBufs + 3) * 8 + 2 * sizeof(StartInfo) + kWeightFloats * 4 + sizeof(EndPlan) <=
                      Cfg::kCtrlBytes,
                  "control block over its bytes");
    int32_t *page_win = reinterpret_cast<int32_t *>(reinterpret_cast<uint8_t *>(merge) +
                                                    kBufs * Cfg::kMergeFloats * 4 + Cfg::kCtrlBytes);

    // A grid queued behind this one (the next call, or the standalone
    // combine) may start its prologue now; it waits for this grid's
    // completion before reading anything.
    grid_dependents_launch();

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], kPaged ? 2 : 1);   // paged caches: the K and the V producer arrive
            mbar_init(&empty[s], kSlices);
        }
        for (int b = 0; b < kBufs; ++b) {
            mbar_init(&mfull[b], kConsumerWarps);
            mbar_init(&mempty[b], kFinisherWarps);
        }
        mbar_init(pbar, 1);
        mbar_init(pbar + 1, 1);
        mbar_init(startbar, 1);
        fence_mbar_init();
    }
    if (warp == kProducerWarp && lane == 0) {   // kernel parameters, not inputs: safe before the wait
        prefetch_tensormap(&tm_k);
        prefetch_tensormap(&tm_v);
        if (kPaged && p.page_shift < 6) {        // small pages: the maps of runs of consecutive pages
            prefetch_tensormap(&tm_kr);
            prefetch_tensormap(&tm_vr);
        }
    }
    // While the previous grid drains (HBM mostly idle), guess this block's
    // first tiles from seqlens as read now and pull them into L2. L2 is the
    // point of coherence, so a stale guess only wastes bandwidth; everything
    // below is recomputed from the real inputs after the wait. The guessed
    // tiles of a contiguous cache are one span of K and one of V (inside the
    // first row), asked for with two bulk prefetches: a tiled prefetch per
    // box costs its issuing thread about as much as a copy, and a block placed
    // late on its SM would otherwise reach the wait late.
    if (!kPaged && warp == 0) {
        find_start<true>(p, guess);
#ifdef FD_DEBUG
        if (lane == 0 && p.debug_spoil_guess) guess->tile = guess->tile > 0 ? guess->tile - 1 : guess->tile + 1;
#endif
        __syncwarp();
        if (lane == 0 && guess->count > 0) {
            const int nt = static_cast<int>(min(static_cast<long long>(kPrefetchTiles),
                                                min(static_cast<long long>(guess->n - guess->tile), guess->count)));
            prefetch_row_span<Cfg::kRowBytes>(p, guess->b * p.Hkv + guess->h, guess->tile, guess->tile + nt);
        }
        __syncwarp();
    }
    __syncthreads();   // barrier inits and the guess are visible to every warp
    // Launched as a programmatic dependent of the previous kernel on the
    // stream: everything above overlaps its tail; inputs are read only after it.
    grid_dependency_wait();
    // The first tiles are issued from the guess (up to one ring's worth,
    // inside the first row) while warp 0 works out the real start from the
    // inputs as they are now: even tiles by the producer, odd ones by
    // finisher warp 9 (idle until the first segment ends), so the two consumer
    // groups' first tiles start at once. When the guess and the real start
    // differ (the lengths changed under the guess), the ring restarts one
    // phase on (below).
    const uint32_t n_spec = !kPaged && guess->count > 0
                                ? static_cast<uint32_t>(min(static_cast<long long>(kStages),
                                                            min(static_cast<long long>(guess->n - guess->tile),
                                                                guess->count)))
                                : 0u;
    if constexpr (!kPaged) if (lane == 0 && (warp == kProducerWarp || warp == kProducerWarp + 1) && n_spec > 0) {
        const uint64_t policy = l2_policy_evict_first();
        const int z = guess->b * p.Hkv + guess->h;
        const uint16_t *q_row =
            p.q + (static_cast<size_t>(guess->b) * p.q_len * p.Hq + static_cast<size_t>(guess->h) * p.g) * D;
        const uint32_t q_run = static_cast<uint32_t>(p.g) * D * 2;
        const uint32_t q_bytes = static_cast<uint32_t>(p.cols) * D * 2;
        // tile t of the first segment into stage t, phase 0
        for (uint32_t t = warp == kProducerWarp ? 0u : 1u; t < n_spec; t += 2) {
            uint8_t *kt = ring + t * Cfg::kStageBytes;
            uint8_t *vt = kt + Cfg::kTileBytes;
            const bool with_q = static_cast<int>(t) < kGroupsC;
            const int y = (guess->tile + static_cast<int>(t)) * kTileTokens;
            mbar_arrive_expect_tx(&full[t], 2 * Cfg::kTileBytes + (with_q ? q_bytes : 0u));
#ifdef FD_DEBUG
            if (blockIdx.x == 0 && static_cast<int>(t) == p.debug_withhold) continue;   // armed, never filled
#endif
            load_tile<Cfg, Consumer::kInterleaved>(kt, vt, &tm_k, &tm_v, &full[t], y, z, policy);
            if (with_q)
                for (int j = 0; j < p.q_len; ++j)
                    bulk_load(vt + Cfg::kTileBytes + j * q_run, q_row + static_cast<size_t>(j) * p.Hq * D, q_run,
                              &full[t]);
        }
    }
    // Warp 0 publishes the real start through an mbarrier rather than a block
    // barrier, so the consumers start on the first tiles while the producer is
    // still issuing.
    if (warp == 0) {
        find_start<false>(p, info);
        if (lane == 0) {
            if (!kPaged && guess->count > 0)
                info->restart = !(info->count == guess->count && info->N == guess->N && info->first == guess->first &&
                                  info->b == guess->b && info->h == guess->h && info->tile == guess->tile &&
                                  info->n == guess->n);
            mbar_arrive(startbar);
        }
    }
    wait_start(startbar);
    // After a wrong guess (the same decision in every thread): the producer lets
    // the guessed copies land (bounded), completes phase 0 of every stage with
    // nothing else in it, and everyone goes on from sequence number kStages
    // (stage s, phase 1). This finishes before any consumer waits on a stage:
    // a wait for phase 1 while phase 0 is still open would pass at once.
    const bool restart = info->restart != 0;
    if (restart) {
        if (warp == kProducerWarp && lane == 0)
            for (int s2 = 0; s2 < kStages; ++s2) {
                if (!kPaged && static_cast<int>(n_spec) > s2)
                    drain_phase(&full[s2], 0);
                else
                    mbar_arrive(&full[s2]);
                mbar_arrive_cnt(&empty[s2], kSlices);
            }
        __syncthreads();
    }

    long long remaining = info->count;
    Cursor c{info->b, info->h, info->tile, info->n, info->first};
    const long long N = info->N;
    volatile int *abort = &info->abort;
    const uint32_t q_bytes = static_cast<uint32_t>(p.cols) * D * 2;   // q_len copies of g rows

    // paged caches: warp 8 brings K and the query heads, warp 11 brings V
    const bool v_role = kPaged && warp == kVProducerWarp;
    if (warp == kProducerWarp || v_role) {
        // ---------------------------------------------------- producer --
        if (lane != 0 || remaining <= 0) return;
        const uint64_t policy = l2_policy_evict_first();
        // paged caches: a window of the current sequence's block-table row in
        // shared memory, fetched with a 1-D bulk copy when a page falls outside
        // it (one window and barrier per producer)
        uint64_t *wbar = pbar + (v_role ? 1 : 0);
        int32_t *win = page_win + (v_role ? kPageWindow : 0);
        int win_b = -1, win_lo = 0, win_hi = 0;
        uint32_t win_phase = 0;
        bool win_pending = false;   // a window copy issued and not yet seen complete
        // page of logical page lp; with need > 1 the window is also made to hold
        // pages lp .. lp + need - 1 (need <= 8, all of them pages of the sequence)
        auto page_of = [&](int b, int lp, int *page, int need = 1) -> bool {
            if (b != win_b || lp < win_lo || lp + need > win_hi) {
                win_b = b;
                win_lo = lp & ~3;
                win_hi = min(win_lo + kPageWindow, p.max_pages);
                const uint32_t bytes = static_cast<uint32_t>(win_hi - win_lo) * 4u;
                mbar_arrive_expect_tx(wbar, bytes);
                if (FD_DCHECK(b < p.B && win_lo >= 0 && win_lo < win_hi))
                    bulk_load(win, p.block_table + static_cast<size_t>(b) * p.max_pages + win_lo, bytes, wbar);
                win_pending = true;
                if (!wait_bounded(wbar, win_phase, abort)) return false;
                win_pending = false;
                win_phase ^= 1u;
            }
            *page = win[lp - win_lo];
            return true;
        };
        // without a restart the guessed tiles already issued are the real first
        // ones: skip them below; after a restart, go on from kStages
        uint32_t seq = restart ? kStages : 0, skip = restart ? 0 : n_spec;
        while (remaining > 0) {
            const int seg = static_cast<int>(min(static_cast<long long>(c.n - c.tile), remaining));
            const int z = c.b * p.Hkv + c.h;
            // query j's g heads: q[b, j, h*g .. h*g+g-1, :], one contiguous run per j
            const uint16_t *q_row =
                p.q + (static_cast<size_t>(c.b) * p.q_len * p.Hq + static_cast<size_t>(c.h) * p.g) * D;
            const uint32_t q_run = static_cast<uint32_t>(p.g) * D * 2;
            const int L = kPaged ? clamp_len(__ldg(p.seqlens + c.b), p.Lmax) : 0;
            for (int k = 0; k < seg; ++k, ++seq) {
                if (seq < skip) continue;   // issued before the barrier, from the guess
                const int stage = static_cast<int>(seq % kStages);
                const uint32_t phase = (seq / kStages) & 1u;
                // once a wait anywhere in the block gave up, issue nothing more (a
                // stage whose copy never completed must not be armed again)
                if (*abort || !wait_bounded(&empty[stage], phase ^ 1u, abort)) {
                    drain_copies<kStages>(full, seq, wbar, win_pending, win_phase);
                    return;
                }
                uint8_t *kt = ring + stage * Cfg::kStageBytes;
                uint8_t *vt = kt + Cfg::kTileBytes;
                const bool with_q = k < kGroupsC && !v_role;   // each group's first tile of the segment
                const uint32_t qb = with_q ? q_bytes : 0u;
#ifdef FD_DEBUG
                if (blockIdx.x == 0 && static_cast<int>(seq) == p.debug_withhold) {
                    // armed, never filled
                    mbar_arrive_expect_tx(&full[stage], (kPaged ? 1 : 2) * Cfg::kTileBytes + qb);
                    continue;
                }
#endif
                const int y = (c.tile + k) * kTileTokens;
                if (!kPaged) {
                    mbar_arrive_expect_tx(&full[stage], 2 * Cfg::kTileBytes + qb);
                    load_tile<Cfg, Consumer::kInterleaved>(kt, vt, &tm_k, &tm_v, &full[stage], y, z, policy);
                } else {
                    // the tile's tokens [y, y + 64) span one page (page_size >= 64) or
                    // 64 / page_size pages; pages past the sequence's end are not loaded
                    // (their rows are masked), so unused block-table entries never matter
                    const int psize = 1 << p.page_shift;
                    const int rows = psize < kTileTokens ? psize : kTileTokens;
                    const int lp0 = y >> p.page_shift;
                    const int npages_seq = (L + psize - 1) >> p.page_shift;
                    const int nsub = psize >= kTileTokens ? 1 : min(kTileTokens >> p.page_shift, npages_seq - lp0);
                    const int off = psize >= kTileTokens ? (y & (psize - 1)) : 0;
                    int page[kTileTokens / 8];
                    int page1 = 0;   // the one page of a tile when page_size >= 64 (kept in a register)
                    if (psize >= kTileTokens) {
                        if (c.b == win_b && lp0 >= win_lo && lp0 < win_hi) {
                            page1 = win[lp0 - win_lo];   // the common case: inside the window
                        } else if (!page_of(c.b, lp0, &page1)) {
                            drain_copies<kStages>(full, seq, wbar, win_pending, win_phase);
                            return;
                        }
                    } else {
                        // the tile's pages lp0 .. lp0 + nsub - 1 (lp0 a multiple of 64 / page_size):
                        // one window check for all of them, then vector loads from the window
                        // (the window starts at a multiple of 4 pages and is 16-byte aligned)
                        if (!(c.b == win_b && lp0 >= win_lo && lp0 + nsub <= win_hi) &&
                            !page_of(c.b, lp0, &page[0], nsub)) {
                            drain_copies<kStages>(full, seq, wbar, win_pending, win_phase);
                            return;
                        }
                        const int* wp = win + (lp0 - win_lo);
                        const int full_tile = kTileTokens >> p.page_shift;
                        if (nsub == full_tile && full_tile >= 4) {
#pragma unroll
                            for (int j4 = 0; j4 < kTileTokens / 8; j4 += 4)
                                if (j4 < nsub) {
                                    const int4 v4 = *reinterpret_cast<const int4 *>(wp + j4);
                                    page[j4] = v4.x;
                                    page[j4 + 1] = v4.y;
                                    page[j4 + 2] = v4.z;
                                    page[j4 + 3] = v4.w;
                                }
                        } else {
#pragma unroll
                            for (int j = 0; j < kTileTokens / 8; ++j)
                                if (j < nsub) page[j] = wp[j];
                        }
                    }
                    // small pages: when the tile's pages are consecutive pages of the pool
                    // (an allocator that hands out pages in order), one box of the run maps
                    // brings them all, with the same bytes at the same places
                    bool run = psize < kTileTokens && nsub == (kTileTokens >> p.page_shift) && page[0] >= 0 &&
                               page[0] <= p.num_pages - nsub;
#pragma unroll
                    for (int j = 1; j < kTileTokens / 8; ++j)
                        if (j < nsub) run = run && page[j] == page[0] + j;
                    const CUtensorMap *rmap = v_role ? &tm_vr : &tm_kr;
                    if constexpr (Consumer::kInterleaved) {
                        // one 5-D box per page, both halves of its tokens: [token][half][128 B].
                        // Coordinates {element, half, token, head, page} (head-major pages)
                        // or {element, half, head, token, page} (token-major pages).
                        const uint32_t page_bytes = static_cast<uint32_t>(rows) * D * 2;
                        mbar_arrive_expect_tx(&full[stage], nsub * page_bytes + qb);
                        const int cz = p.kv_nhd ? c.h : off, cw = p.kv_nhd ? off : c.h;
                        const CUtensorMap *map = v_role ? &tm_v : &tm_k;
                        uint8_t *dst = v_role ? vt : kt;
                        if (run)   // box {64, 2, page_size, 1, nsub} (head-major) or {64, 2, 1, page_size, nsub}
                            tma_load_5d(dst, rmap, &full[stage], 0, 0, cz, cw, page[0], policy);
                        else   // (a loop with constant indices measured slower here, unlike the 3-D boxes below)
                            for (int j = 0; j < nsub; ++j)
                                tma_load_5d(dst + j * page_bytes, map, &full[stage], 0, 0, cz, cw, page[j], policy);
                    } else {
                        // a page's rows of one box column land at j * rows box rows
                        const uint32_t sub_bytes = static_cast<uint32_t>(rows) * Cfg::kBoxRowBytes;
                        mbar_arrive_expect_tx(&full[stage], nsub * sub_bytes * Cfg::kBoxes + qb);
                        const CUtensorMap *map = v_role ? &tm_v : &tm_k;
                        uint8_t *dstb = v_role ? vt : kt;
                        if (run) {
                            // run maps: {element, token, head, page} with box {cols, page_size, 1, nsub}
                            // (head-major) or {element, head, page * page_size + token} with box
                            // {cols, 1, 64} (token-major): page j's rows land at j * rows box rows
#pragma unroll
                            for (int bx = 0; bx < Cfg::kBoxes; ++bx) {
                                const int x = Cfg::kBoxCols * bx;
                                if (p.kv_nhd)
                                    tma_load_3d(dstb + bx * Cfg::kBoxBytes, rmap, &full[stage], x, c.h,
                                                page[0] << p.page_shift, policy);
                                else
                                    tma_load_4d(dstb + bx * Cfg::kBoxBytes, rmap, &full[stage], x, 0, c.h, page[0],
                                                policy);
                            }
                        } else
#pragma unroll
                        for (int j = 0; j < kTileTokens / 8; ++j) {   // constant indices: page[] stays in registers
                            if (j >= nsub) break;
                            const int pgj = psize >= kTileTokens ? page1 : page[j];
#pragma unroll
                            for (int bx = 0; bx < Cfg::kBoxes; ++bx) {
                                const int dst = bx * Cfg::kBoxBytes + j * rows * Cfg::kBoxRowBytes;
                                const int x = Cfg::kBoxCols * bx;
                                // 3-D page maps: {element, token, page * Hkv + head} (head-major)
                                // or {element, head, page * page_size + token} (token-major)
                                // a page outside the pool gets a coordinate outside the tensor (zeros)
                                const bool inside = pgj >= 0 && pgj < p.num_pages;
                                if (p.kv_nhd) {
                                    const int zz = inside ? pgj * (1 << p.page_shift) + off : -kTileTokens;
                                    tma_load_3d(dstb + dst, map, &full[stage], x, c.h, zz, policy);
                                } else {
                                    const int zz = inside ? pgj * p.Hkv + c.h : -1;
                                    tma_load_3d(dstb + dst, map, &full[stage], x, off, zz, policy);
                                }
                            }
                        }
                    }
                }
                if (with_q)
                    for (int j = 0; j < p.q_len; ++j) {
                        const uint16_t *src = q_row + static_cast<size_t>(j) * p.Hq * D;
                        if (FD_DCHECK(src >= p.q && src + q_run / 2 <= p.q + out_rows(p) * D))
                            bulk_load(vt + Cfg::kTileBytes + j * q_run, src, q_run, &full[stage]);
                    }
            }
            remaining -= seg;
            if (remaining > 0) next_row(c, p);
        }
        // after an abort the consumers no longer wait for the last stages: the
        // producer keeps the block alive until its copies have landed
        if (*abort) drain_copies<kStages>(full, seq, wbar, win_pending, win_phase);
        return;
    }

    Cursor last_c = c;          // the run's last segment: merged by all workers at the end
    int last_seg = 0;
    if (warp < kConsumerWarps) {
        // ---------------------------------------------------- consumers --
        const int group = warp / kSlices, slice = warp % kSlices;
        Consumer cons;
        cons.init(p);
        uint32_t seq = restart ? kStages : 0, segctr = 0;
        while (remaining > 0) {
            const int seg = static_cast<int>(min(static_cast<long long>(c.n - c.tile), remaining));
            const int L = clamp_len(__ldg(p.seqlens + c.b), p.Lmax);
            cons.reset();
            cons.set_row(p, c.h);
            for (int k = 0; k < seg; ++k, ++seq) {
                if (static_cast<int>(seq % kGroupsC) != group) continue;
                const int stage = static_cast<int>(seq % kStages);
                const uint32_t phase = (seq / kStages) & 1u;
                wait_bounded(&full[stage], phase, abort);   // on abort: keep going, outputs are flagged invalid
                const uint8_t *st = ring + stage * Cfg::kStageBytes;
                if (k < kGroupsC) cons.load_q(st + 2 * Cfg::kTileBytes, p.cols);
                const uint32_t kt = smem_addr(st);
                const int valid = L - ((c.tile + k) * kTileTokens + kTok * slice);
                cons.tile(kt, kt + Cfg::kTileBytes, slice, valid, p.scale_log2e);
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[stage]);
            }
            // hand this segment's state to the finishers and go on
            const int buf = static_cast<int>(segctr % kBufs);
            wait_bounded(&mempty[buf], ((segctr / kBufs) & 1u) ^ 1u, abort);
            cons.to_smem(merge + buf * Cfg::kMergeFloats + warp * Cfg::kWarpFloats);
            __syncwarp();
            if (lane == 0) mbar_arrive(&mfull[buf]);
            if (tid == 0) info->last_buf = buf;
            ++segctr;
            last_c = c;
            last_seg = seg;
            remaining -= seg;
            if (remaining > 0) next_row(c, p);
        }
    } else {
        // ---------------------------------------------------- finishers --
        const int ftid = tid - (kProducerWarp + 1) * 32;
        if (kFused) {
            // rows without tokens (no segment, no ticket): out = 0, lse = -inf,
            // written by block u % P while the first tiles are on their way
            for (long long u = blockIdx.x; u < static_cast<long long>(p.B) * p.Hkv; u += p.P) {
                const int b = static_cast<int>(u / p.Hkv), h = static_cast<int>(u % p.Hkv);
                if (clamp_len(__ldg(p.seqlens + b), p.Lmax) != 0) continue;
                for (int idx = ftid; idx < p.cols * (D / 4); idx += kFinisherThreads) {
                    const int col = idx / (D / 4), d4 = idx - col * (D / 4);
                    const size_t row = out_row(p, b, h, col);
                    if (!FD_DCHECK(row < out_rows(p))) continue;
                    reinterpret_cast<float4 *>(p.out + row * D)[d4] = make_float4(0.f, 0.f, 0.f, 0.f);
                    if (d4 == 0) p.lse[row] = -INFINITY;
                }
            }
        }
        uint32_t segctr = 0;
        while (remaining > 0) {
            const int seg = static_cast<int>(min(static_cast<long long>(c.n - c.tile), remaining));
            if (seg == remaining) {   // the last segment: left for all workers at the end
                last_c = c;
                last_seg = seg;
                if (kFused && ftid == 0) info->last_rr = row_runs(c.first, c.n, N, p.P);   // ahead of its ticket
                break;
            }
            const bool whole = c.tile == 0 && seg == c.n;
            const long long u = static_cast<long long>(c.b) * p.Hkv + c.h;
            const size_t slot = static_cast<size_t>(blockIdx.x) + static_cast<size_t>(u);
            const int buf = static_cast<int>(segctr % kBufs);
            wait_bounded(&mfull[buf], (segctr / kBufs) & 1u, abort);
            merge_warps_and_store<D, G>(merge + buf * Cfg::kMergeFloats, weights, p, c, whole, slot, ftid,
                                        kFinisherThreads, [] { named_barrier_sync(kBarFinishers, kFinisherThreads); });
            named_barrier_sync(kBarFinishers, kFinisherThreads);   // every finisher is done with the buffer
            if (lane == 0) mbar_arrive(&mempty[buf]);
            // the barrier above orders every finisher's stores before the ticket
            if (kFused && !whole && ftid == 0)
                take_ticket<D>(p, info, plan, c, row_runs(c.first, c.n, N, p.P), N, kStageFloats);
            ++segctr;
            remaining -= seg;
            if (remaining > 0) next_row(c, p);
        }
    }

    // ------------------------------------------ end of the run (all but the producer) --
    // The consumers have dumped the last segment; the finishers have stored
    // every earlier one. All 320 threads merge and store the last segment.
    const int wtid = tid < kConsumerThreads ? tid : tid - 32;   // skip the producer warp
    auto workers_sync = [] { named_barrier_sync(kBarWorkers, kWorkerThreads); };
    workers_sync();
    if (info->count > 0) {
        const bool whole = last_c.tile == 0 && last_seg == last_c.n;
        const long long u = static_cast<long long>(last_c.b) * p.Hkv + last_c.h;
        const size_t slot = static_cast<size_t>(blockIdx.x) + static_cast<size_t>(u);
        const int buf = static_cast<int>(info->last_buf);
        merge_warps_and_store<D, G>(merge + buf * Cfg::kMergeFloats, weights, p, last_c, whole, slot, wtid,
                                    kWorkerThreads, workers_sync);
        if (kFused && !whole) {
            workers_sync();   // the stores above, before the ticket
            if (wtid == 0) take_ticket<D>(p, info, plan, last_c, info->last_rr, N, kStageFloats);
        }
        workers_sync();
    }
    if (kFused) {
        // Everything this block's tickets completed, with every worker:
        //  1. chunks of two-level rows: merge the chunk's segments (at most
        //     kFanIn: one L2 round trip) into its partial, written over the
        //     slot of the chunk's first segment, then take the row's ticket;
        //  2. complete rows: fold their units (segments, or the chunks'
        //     partials) in order. Few units are read straight from L2 (one
        //     round trip); more are staged in the ring and merge buffers (all
        //     free now) with every copy in flight at once, as many rows
        //     together as fit, and folded from there; a row too large to
        //     stage is read from L2.
        // One float4 output per thread and step throughout.
        constexpr int kVec = D / 4;
        float *staged = reinterpret_cast<float *>(ring);
        const int row_vec = p.cols * kVec;
        auto entry_ok = [&](int k) {   // the entry's outputs and units lie inside their buffers
            return FD_DCHECK(out_row(p, info->pending[k].b, info->pending[k].h, p.cols - 1) < out_rows(p) &&
                             (plan->m[k].slot0 + static_cast<size_t>(plan->m[k].count - 1) * plan->m[k].stride + 1) *
                                     p.cols <=
                                 seg_rows(p));
        };
        auto store = [&](int k, int head, int d4, float4 v, float lse) {
            const size_t row = out_row(p, info->pending[k].b, info->pending[k].h, head);
            reinterpret_cast<float4 *>(p.out + row * D)[d4] = v;
            if (d4 == 0) p.lse[row] = lse;
        };

        // (every entry and its plan were written before the last barrier)
        int npending = *reinterpret_cast<volatile int *>(&info->npending);
        bool any_chunk = false;
        for (int k = 0; k < npending; ++k) any_chunk |= plan->mode[k] == kEndChunk;
        if (any_chunk) {
            // 1. outputs first; a chunk's lse is written only after the barrier,
            //    since every thread of a head reads the lse slot it overwrites
            for (int idx = wtid; idx < npending * row_vec; idx += kWorkerThreads) {
                const int k = idx / row_vec, rem = idx - k * row_vec;
                if (plan->mode[k] != kEndChunk || !entry_ok(k)) continue;
                const Units m = plan->m[k];
                const int head = rem / kVec, d4 = rem % kVec;
                float lse;
                const float4 v =
                    merge_l2<D, 1>(p.seg_out, p.seg_lse, p.cols, m.slot0, m.count, m.i0, m.i1, N, p.P, head, d4, &lse);
                reinterpret_cast<float4 *>(p.seg_out + (m.slot0 * p.cols + head) * D)[d4] = v;
                if (d4 == 0) staged[k * p.cols + head] = lse;
            }
            workers_sync();
            for (int v = wtid; v < npending * p.cols; v += kWorkerThreads) {
                const int k = v / p.cols, head = v - k * p.cols;
                if (plan->mode[k] != kEndChunk || !entry_ok(k)) continue;
                const size_t slot0 = plan->m[k].slot0;
                p.seg_lse[slot0 * p.cols + head] = staged[v];
                if (head == 0) p.chunk_tickets[slot0] = 0;   // every segment of the chunk has arrived
            }
            workers_sync();   // the partials, before their row's ticket
            if (wtid == 0) {
                const int n0 = npending;
                for (int k = 0; k < n0; ++k) {
                    if (plan->mode[k] != kEndChunk) continue;
                    const PendingRow r = info->pending[k];
                    const long long u = static_cast<long long>(r.b) * p.Hkv + r.h;
                    if (!FD_DCHECK(u < static_cast<long long>(p.B) * p.Hkv)) continue;
                    const int prev = atom_add_acq_rel_gpu(p.row_tickets + u, 1);
                    if (prev == row_chunk_count(r.rr, N, p.P) - 1)
                        queue_pending<D>(p, info, plan, r.b, r.h, -1, r.rr, kStageFloats);
                }
            }
            workers_sync();
            npending = *reinterpret_cast<volatile int *>(&info->npending);
        }

        // 2. complete rows: the direct ones together (one round trip for all)
        for (int idx = wtid; idx < npending * row_vec; idx += kWorkerThreads) {
            const int k = idx / row_vec, rem = idx - k * row_vec;
            if (plan->mode[k] != kEndDirect || !entry_ok(k)) continue;
            const int head = rem / kVec, d4 = rem % kVec;
            const Units m = plan->m[k];
            float lse;
            const float4 v = merge_units_l2<D>(p.seg_out, p.seg_lse, p.cols, m, N, p.P, head, d4, &lse);
            store(k, head, d4, v, lse);
        }
        for (int k = 0; k < npending; ++k) {   // too large to stage
            if (plan->mode[k] != kEndFromL2 || !entry_ok(k)) continue;
            const Units m = plan->m[k];
            for (int idx = wtid; idx < row_vec; idx += kWorkerThreads) {
                const int head = idx / kVec, d4 = idx % kVec;
                float lse;
                const float4 v = merge_units_l2<D>(p.seg_out, p.seg_lse, p.cols, m, N, p.P, head, d4, &lse);
                store(k, head, d4, v, lse);
            }
        }
        int i = 0;   // staged rows, as many together as fit
        while (i < npending) {
            if (plan->mode[i] != kEndStaged) {
                ++i;
                continue;
            }
            int j = i;
            long long used = 0;
            while (j < npending) {
                const long long need =
                    plan->mode[j] == kEndStaged ? staged_floats(plan->m[j].count, p.cols, D) : 0;
                if (used + need > kStageFloats) break;
                used += need;
                ++j;
            }
            long long off = 0;
            for (int k = i; k < j; ++k) {
                if (plan->mode[k] != kEndStaged) continue;
                if (entry_ok(k)) stage_units<D>(staged + off, p.seg_out, p.seg_lse, p.cols, plan->m[k], wtid, kWorkerThreads);
                off += staged_floats(plan->m[k].count, p.cols, D);
            }
            cp_async_wait_all();
            workers_sync();
            off = 0;
            for (int k = i; k < j; ++k) {
                if (plan->mode[k] != kEndStaged) continue;
                if (entry_ok(k)) {
                    const Units m = plan->m[k];
                    for (int idx = wtid; idx < row_vec; idx += kWorkerThreads) {
                        const int head = idx / kVec, d4 = idx % kVec;
                        float lse;
                        const float4 v = merge_staged_vec<D>(staged + off, p.cols, m, N, p.P, head, d4, &lse);
                        store(k, head, d4, v, lse);
                    }
                }
                off += staged_floats(plan->m[k].count, p.cols, D);
            }
            workers_sync();   // before the next rows are staged over these
            i = j;
        }
        if (wtid < npending && plan->mode[wtid] != kEndChunk) {   // every unit has arrived: reset for the next call
            const PendingRow r = info->pending[wtid];
            p.row_tickets[static_cast<long long>(r.b) * p.Hkv + r.h] = 0;
        }
    }
}

}  // namespace fd
