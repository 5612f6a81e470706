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
    r.count = r.i1 - r.i0 + 1;
    if (N < P)
        for (int i = r.i0; i <= r.i1; ++i) r.count -= run_is_empty(i, N, P) ? 1 : 0;
    return r;
}

// One float4 of the merged output of a row: head `head`, columns 4*d4..4*d4+3.
// Walks the segments once, in slot order, with a running maximum
//     M <- max(M, lse_s);  S = sum exp(lse_s - M);  acc = sum exp(lse_s - M) O_s
// and returns acc / S (and LSE = M + log S through *lse). Loads are issued
// eight segments at a time before any of them is used, so a row costs one L2
// round trip per eight segments. Reads go to L2 (.cg): the segments were
// written by other blocks of the same grid.
template <int D>
__device__ __forceinline__ float4 merge_row_vec(const float *seg_out, const float *seg_lse, int g, size_t slot0,
                                                int nseg, int i0, long long N, int P, int head, int d4,
                                                float *lse) {
    constexpr int kChunk = 8;
    const bool maybe_empty = N < P;
    float M = -INFINITY, S = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int s0 = 0; s0 < nseg; s0 += kChunk) {
        float ls[kChunk];
        float4 o[kChunk];
#pragma unroll
        for (int j = 0; j < kChunk; ++j) {
            const int s = s0 + j;
            ls[j] = -INFINITY;
            o[j] = make_float4(0.f, 0.f, 0.f, 0.f);
            if (s < nseg && !(maybe_empty && run_is_empty(i0 + s, N, P))) {
                const size_t r = (slot0 + s) * g + head;
                ls[j] = __ldcg(seg_lse + r);
                o[j] = __ldcg(reinterpret_cast<const float4 *>(seg_out + r * D) + d4);
            }
        }
#pragma unroll
        for (int j = 0; j < kChunk; ++j) {
            if (ls[j] == -INFINITY) continue;
            if (ls[j] > M) {   // new maximum: rescale what has been summed so far
                const float c = ex2((M - ls[j]) * kLog2eF);
                S *= c;
                acc.x *= c;
                acc.y *= c;
                acc.z *= c;
                acc.w *= c;
                M = ls[j];
            }
            const float w = ex2((ls[j] - M) * kLog2eF);
            S += w;
            acc.x = fmaf(w, o[j].x, acc.x);
            acc.y = fmaf(w, o[j].y, acc.y);
            acc.z = fmaf(w, o[j].z, acc.z);
            acc.w = fmaf(w, o[j].w, acc.w);
        }
    }
    if (M == -INFINITY) {
        *lse = -INFINITY;
        return make_float4(0.f, 0.f, 0.f, 0.f);
    }
    const float inv = 1.f / S;
    *lse = M + lg2(S) * kLn2F;
    return make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
}

// Merge row u's segments into out_row[g][D] / lse_row[g] with `nthreads`
// threads (tid = 0..nthreads-1), one float4 output per thread and step.
template <int D>
__device__ __forceinline__ void merge_row(const float *seg_out, const float *seg_lse, int g, long long u,
                                          const RowRuns &rr, long long N, int P, float *out_row, float *lse_row,
                                          int tid, int nthreads) {
    const int nseg = rr.i1 - rr.i0 + 1;
    const size_t slot0 = static_cast<size_t>(rr.i0) + static_cast<size_t>(u);
    constexpr int kVec = D / 4;
    for (int idx = tid; idx < g * kVec; idx += nthreads) {
        const int head = idx / kVec, d4 = idx - head * kVec;
        float lse;
        const float4 v = merge_row_vec<D>(seg_out, seg_lse, g, slot0, nseg, rr.i0, N, P, head, d4, &lse);
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
