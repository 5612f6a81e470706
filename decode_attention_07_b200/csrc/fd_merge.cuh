// fd_merge.cuh -- the final reduction of one row over its segments.
//
// "Flash-Decoding for long-context inference", section "A faster attention
// for decoding: Flash-Decoding": the output is obtained by reducing over all
// splits, each split's contribution scaled through its log-sum-exp. For one
// row with segments s (normalised outputs O_s, natural-log lse_s):
//     LSE = M + log sum_s exp(lse_s - M),   M = max_s lse_s
//     out = sum_s exp(lse_s - LSE) * O_s    (s in increasing order)
// Used by the split kernel's last block on a row (in-kernel combine) and by
// the standalone combine kernel, so both produce bitwise the same values.
//
// A row cut into more than kTwoLevelSegs segments, or whose segments would
// not fit the shared memory a block has free at the end of its run
// (kStageBudgetFloats), is reduced in two levels
// (the same formula applied to groups, which the formula allows: merging
// merged groups gives the merge of all): its segments are taken kFanIn at a
// time in slot order ("chunks"), each chunk is merged into one partial
// (O_c, lse_c), and the chunks' partials are merged in order into the row.
// With one block completing a row, this spreads a long row's reduction over
// the blocks that complete its chunks instead of one block reading every
// segment.
#pragma once

#include "fd_partition.cuh"
#include "fd_ptx.cuh"

namespace fd {

constexpr float kLog2eF = 1.44269504088896341f;
constexpr float kLn2F = 0.693147180559945309f;

// Segment slots of row u are i + u for runs i in [i0, i1]; with more runs
// than tiles (N < P) some of those runs are empty and wrote nothing.
__device__ __forceinline__ bool run_is_empty(int i, long long N, int P) {
    return run_begin(i, N, P) == run_begin(i + 1, N, P);
}

// Segments of the row whose first flat tile is `first` and which has n tiles.
struct RowRuns {
    int i0, i1, count;   // first / last run touching the row, runs that hold tiles of it
};

__device__ __forceinline__ RowRuns row_runs(long long first, int n, long long N, int P) {
    RowRuns r;
    r.i0 = run_of_tile(first, N, P);
    r.i1 = run_of_tile(first + n - 1, N, P);
    // with more runs than tiles every run holds at most one tile, so the
    // runs holding the row's n tiles are n distinct ones
    r.count = N < P ? n : r.i1 - r.i0 + 1;
    return r;
}

// The running merge of one float4 of a row over its segments, in slot order:
//     M <- max(M, lse_s);  S = sum exp(lse_s - M);  acc = sum exp(lse_s - M) O_s
// and at the end out = acc / S, LSE = M + log S. Every merge of segments
// (from L2, from shared memory, in either kernel) goes through these steps,
// so all of them give bitwise the same values.
struct MergeState {
    float M, S;
    float4 acc;
};

__device__ __forceinline__ MergeState merge_begin() {
    MergeState st;
    st.M = -INFINITY;
    st.S = 0.f;
    st.acc = make_float4(0.f, 0.f, 0.f, 0.f);
    return st;
}

// Fold one segment (lse ls, normalised output o) in; ls = -inf weighs nothing.
__device__ __forceinline__ void merge_fold(MergeState &st, float ls, const float4 &o) {
    if (ls == -INFINITY) return;
    if (ls > st.M) {   // new maximum: rescale what has been summed so far
        const float c = ex2((st.M - ls) * kLog2eF);
        st.S *= c;
        st.acc.x *= c;
        st.acc.y *= c;
        st.acc.z *= c;
        st.acc.w *= c;
        st.M = ls;
    }
    const float w = ex2((ls - st.M) * kLog2eF);
    st.S += w;
    st.acc.x = fmaf(w, o.x, st.acc.x);
    st.acc.y = fmaf(w, o.y, st.acc.y);
    st.acc.z = fmaf(w, o.z, st.acc.z);
    st.acc.w = fmaf(w, o.w, st.acc.w);
}

// acc / S and LSE (through *lse); no segment with tokens: 0 and -inf.
__device__ __forceinline__ float4 merge_end(const MergeState &st, float *lse) {
    if (st.M == -INFINITY) {
        *lse = -INFINITY;
        return make_float4(0.f, 0.f, 0.f, 0.f);
    }
    const float inv = 1.f / st.S;
    *lse = st.M + lg2(st.S) * kLn2F;
    return make_float4(st.acc.x * inv, st.acc.y * inv, st.acc.z * inv, st.acc.w * inv);
}

constexpr int kFanIn = 8;            // segments per chunk of a two-level row
constexpr int kTwoLevelSegs = 64;    // rows with more segment slots are reduced in two levels
// Rows whose segments take more floats than this staged (outputs and lse)
// are reduced in two levels too. Every split-kernel configuration that runs
// more than one column has more shared memory free at the end of its run
// (its ring and merge buffers); one column never gets near it.
constexpr long long kStageBudgetFloats = 160 * 1024 / 4;

__device__ __forceinline__ int row_slots(const RowRuns &rr) { return rr.i1 - rr.i0 + 1; }
// Floats a merge's units take when staged in shared memory by stage_units:
// outputs [count][g][D], then the lse values [count][g] padded to a multiple
// of four (the next staged merge starts 16-byte aligned).
__device__ __forceinline__ long long staged_floats(int count, int g, int D) {
    const long long n = static_cast<long long>(count) * g;
    return n * D + ((n + 3) & ~3LL);
}

// g: columns per row (query heads per kv head, times queries per sequence).
__device__ __forceinline__ bool is_two_level(const RowRuns &rr, int g, int D) {
    return row_slots(rr) > kTwoLevelSegs || staged_floats(row_slots(rr), g, D) > kStageBudgetFloats;
}
__device__ __forceinline__ int num_chunks(const RowRuns &rr) { return (row_slots(rr) + kFanIn - 1) / kFanIn; }

// Runs of chunk c that hold tiles of the row: the chunk's ticket count.
__device__ __forceinline__ int chunk_count(const RowRuns &rr, int c, long long N, int P) {
    const int a = rr.i0 + c * kFanIn, b = min(rr.i1, a + kFanIn - 1);
    int n = b - a + 1;
    if (N < P)
        for (int i = a; i <= b; ++i) n -= run_is_empty(i, N, P) ? 1 : 0;
    return n;
}

// Chunks holding tiles: the row ticket count of a two-level row.
__device__ __forceinline__ int row_chunk_count(const RowRuns &rr, long long N, int P) {
    const int nc = num_chunks(rr);
    if (N >= P) return nc;
    int n = 0;
    for (int c = 0; c < nc; ++c) n += chunk_count(rr, c, N, P) > 0 ? 1 : 0;
    return n;
}

// The units one merge folds, in order: unit s sits in slot slot0 + s*stride.
// Runs i0..i1 are the runs those units cover.
struct Units {
    size_t slot0;
    int stride, count;
    int i0, i1;
};

// The segments of row u (single level), or of its chunk c (first level).
__device__ __forceinline__ Units segment_units(const RowRuns &rr, long long u) {
    return Units{static_cast<size_t>(rr.i0) + static_cast<size_t>(u), 1, row_slots(rr), rr.i0, rr.i1};
}
__device__ __forceinline__ Units chunk_units(const RowRuns &rr, long long u, int c) {
    const int a = rr.i0 + c * kFanIn, b = min(rr.i1, a + kFanIn - 1);
    return Units{static_cast<size_t>(a) + static_cast<size_t>(u), 1, b - a + 1, a, b};
}
// The chunks' partials of a two-level row (second level): chunk c's partial
// is kept in the slot of the chunk's first segment.
__device__ __forceinline__ Units partial_units(const RowRuns &rr, long long u) {
    return Units{static_cast<size_t>(rr.i0) + static_cast<size_t>(u), kFanIn, num_chunks(rr), rr.i0, rr.i1};
}
// What the last reduction of a row folds.
__device__ __forceinline__ Units final_units(const RowRuns &rr, long long u, int g, int D) {
    return is_two_level(rr, g, D) ? partial_units(rr, u) : segment_units(rr, u);
}

// Runs a..b (a chunk) hold no tile: only possible with more runs than tiles.
__device__ __forceinline__ bool runs_empty(int a, int b, long long N, int P) {
    for (int i = a; i <= b; ++i)
        if (!run_is_empty(i, N, P)) return false;
    return true;
}

// Unit s holds nothing: an empty run, or a chunk of empty runs (only with
// more runs than tiles).
__device__ __forceinline__ bool unit_empty(const Units &m, int s, long long N, int P) {
    if (N >= P) return false;
    if (m.stride == 1) return run_is_empty(m.i0 + s, N, P);
    const int a = m.i0 + s * m.stride;
    return runs_empty(a, min(m.i1, a + m.stride - 1), N, P);
}

// One float4 of a merge read from L2: `count` units in slots slot0,
// slot0 + kStride, ... (kStride = 1: segments of runs i0, i0 + 1, ...;
// kStride = kFanIn: chunk partials), head `head`, columns 4*d4..4*d4+3.
// Loads are issued eight units at a time before any of them is used, so a
// merge costs one L2 round trip per eight units. Reads go to L2 (.cg): the
// units were written by other blocks of the same grid.
template <int D, int kStride>
__device__ __forceinline__ float4 merge_l2(const float *seg_out, const float *seg_lse, int g, size_t slot0, int count,
                                           int i0, int i1, long long N, int P, int head, int d4, float *lse) {
    constexpr int kBatch = 8;
    const bool maybe_empty = N < P;
    MergeState st = merge_begin();
    for (int s0 = 0; s0 < count; s0 += kBatch) {
        float ls[kBatch];
        float4 o[kBatch];
#pragma unroll
        for (int j = 0; j < kBatch; ++j) {
            const int s = s0 + j;
            ls[j] = -INFINITY;
            o[j] = make_float4(0.f, 0.f, 0.f, 0.f);
            const bool empty =
                maybe_empty && (kStride == 1 ? run_is_empty(i0 + s, N, P)
                                             : runs_empty(i0 + s * kStride, min(i1, i0 + s * kStride + kStride - 1), N, P));
            if (s < count && !empty) {
                const size_t r = (slot0 + static_cast<size_t>(s) * kStride) * g + head;
                ls[j] = __ldcg(seg_lse + r);
                o[j] = __ldcg(reinterpret_cast<const float4 *>(seg_out + r * D) + d4);
            }
        }
#pragma unroll
        for (int j = 0; j < kBatch; ++j) merge_fold(st, ls[j], o[j]);
    }
    return merge_end(st, lse);
}

// merge_l2 over the units of m.
template <int D>
__device__ __forceinline__ float4 merge_units_l2(const float *seg_out, const float *seg_lse, int g, const Units &m,
                                                 long long N, int P, int head, int d4, float *lse) {
    return m.stride == 1
               ? merge_l2<D, 1>(seg_out, seg_lse, g, m.slot0, m.count, m.i0, m.i1, N, P, head, d4, lse)
               : merge_l2<D, kFanIn>(seg_out, seg_lse, g, m.slot0, m.count, m.i0, m.i1, N, P, head, d4, lse);
}

// One float4 of a whole row's reduction straight from its segments in L2,
// two-level rows included (each chunk merged, then folded in as a partial):
// the standalone combine's path, and bitwise what the fused path computes.
template <int D>
__device__ __forceinline__ float4 merge_row_vec(const float *seg_out, const float *seg_lse, int g, long long u,
                                                const RowRuns &rr, long long N, int P, int head, int d4,
                                                float *lse) {
    const size_t slot0 = static_cast<size_t>(rr.i0) + static_cast<size_t>(u);
    if (!is_two_level(rr, g, D))
        return merge_l2<D, 1>(seg_out, seg_lse, g, slot0, row_slots(rr), rr.i0, rr.i1, N, P, head, d4, lse);
    MergeState row = merge_begin();
    const int nc = num_chunks(rr);
    for (int c = 0; c < nc; ++c) {
        const int a = rr.i0 + c * kFanIn, b = min(rr.i1, a + kFanIn - 1);
        if (N < P && runs_empty(a, b, N, P)) continue;
        float lc;
        const float4 oc = merge_l2<D, 1>(seg_out, seg_lse, g, slot0 + static_cast<size_t>(c) * kFanIn, b - a + 1, a, b,
                                         N, P, head, d4, &lc);
        merge_fold(row, lc, oc);
    }
    return merge_end(row, lse);
}

// Copy a merge's units to shared memory at dst, spread over `nthreads`
// threads: outputs by cp.async, 16 bytes each and all in flight at once,
// the lse values by plain L2 loads. The caller completes the copies
// (cp_async_wait_all) and syncs before reading them.
template <int D>
__device__ __forceinline__ void stage_units(float *dst, const float *seg_out, const float *seg_lse, int g,
                                            const Units &m, int tid, int nthreads) {
    const int per = g * (D / 4);   // float4s per unit
    const int nvec = m.count * per;
    const float4 *src = reinterpret_cast<const float4 *>(seg_out) + m.slot0 * per;
    float4 *d = reinterpret_cast<float4 *>(dst);
    float *dl = dst + static_cast<size_t>(m.count) * g * D;
    const float *sl = seg_lse + m.slot0 * g;
    if (m.stride == 1) {   // consecutive slots: one contiguous range
        for (int v = tid; v < nvec; v += nthreads) cp_async_16(d + v, src + v);
        for (int v = tid; v < m.count * g; v += nthreads) dl[v] = __ldcg(sl + v);
    } else {
        for (int v = tid; v < nvec; v += nthreads) {
            const int s = v / per, w = v - s * per;
            cp_async_16(d + v, src + static_cast<size_t>(s) * m.stride * per + w);
        }
        for (int v = tid; v < m.count * g; v += nthreads) {
            const int s = v / g, h = v - s * g;
            dl[v] = __ldcg(sl + static_cast<size_t>(s) * m.stride * g + h);
        }
    }
}

// One float4 of a merge staged by stage_units: the same folds, in the same
// order, as merge_units_l2.
template <int D>
__device__ __forceinline__ float4 merge_staged_vec(const float *staged, int g, const Units &m, long long N, int P,
                                                   int head, int d4, float *lse) {
    const float4 *o = reinterpret_cast<const float4 *>(staged);
    const float *ls = staged + static_cast<size_t>(m.count) * g * D;
    MergeState st = merge_begin();
    for (int s = 0; s < m.count; ++s) {
        if (unit_empty(m, s, N, P)) continue;
        merge_fold(st, ls[s * g + head], o[(s * g + head) * (D / 4) + d4]);
    }
    return merge_end(st, lse);
}

// Merge row u's segments into out_row[g][D] / lse_row[g] with `nthreads`
// threads (tid = 0..nthreads-1), one float4 output per thread and step.
template <int D>
__device__ __forceinline__ void merge_row(const float *seg_out, const float *seg_lse, int g, long long u,
                                          const RowRuns &rr, long long N, int P, float *out_row, float *lse_row,
                                          int tid, int nthreads) {
    constexpr int kVec = D / 4;
    for (int idx = tid; idx < g * kVec; idx += nthreads) {
        const int head = idx / kVec, d4 = idx - head * kVec;
        float lse;
        const float4 v = merge_row_vec<D>(seg_out, seg_lse, g, u, rr, N, P, head, d4, &lse);
        reinterpret_cast<float4 *>(out_row + head * D)[d4] = v;
        if (d4 == 0) lse_row[head] = lse;
    }
}

// Rows with no tokens: out = 0, lse = -inf.
template <int D>
__device__ __forceinline__ void write_empty_row(float *out_row, float *lse_row, int g, int tid, int nthreads) {
    for (int idx = tid; idx < g * (D / 4); idx += nthreads) {
        reinterpret_cast<float4 *>(out_row)[idx] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (idx % (D / 4) == 0) lse_row[idx / (D / 4)] = -INFINITY;
    }
}

}  // namespace fd
