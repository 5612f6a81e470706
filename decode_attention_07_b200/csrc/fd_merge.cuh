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

// Merge row u's segments into out_row[g][D] / lse_row[g]. Called by `nthreads`
// threads (tid = 0..nthreads-1, whole warps) that share `s_lse` (>= g floats
// of shared memory) and the barrier `bar`. Reads go to L2 (.cg): the segments
// were written by other blocks of the same grid.
template <int D, class Bar>
__device__ __forceinline__ void merge_row(const float *seg_out, const float *seg_lse, int g, long long u,
                                          const RowRuns &rr, long long N, int P, float *out_row, float *lse_row,
                                          float *s_lse, int tid, int nthreads, Bar bar) {
    const int lane = tid & 31, warp = tid >> 5, nwarps = nthreads >> 5;
    const int nseg = rr.i1 - rr.i0 + 1;
    const size_t slot0 = static_cast<size_t>(rr.i0) + static_cast<size_t>(u);
    const bool maybe_empty = N < P;

    for (int head = warp; head < g; head += nwarps) {
        float mx = -INFINITY;
        for (int s = lane; s < nseg; s += 32)
            if (!maybe_empty || !run_is_empty(rr.i0 + s, N, P))
                mx = fmaxf(mx, __ldcg(seg_lse + (slot0 + s) * g + head));
        for (int sh = 16; sh > 0; sh >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, sh));
        float sum = 0.f;
        if (mx != -INFINITY)
            for (int s = lane; s < nseg; s += 32)
                if (!maybe_empty || !run_is_empty(rr.i0 + s, N, P))
                    sum += ex2((__ldcg(seg_lse + (slot0 + s) * g + head) - mx) * kLog2eF);
        for (int sh = 16; sh > 0; sh >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, sh);
        if (lane == 0) s_lse[head] = mx == -INFINITY ? -INFINITY : mx + lg2(sum) * kLn2F;
    }
    bar();

    constexpr int kVec = D / 4;   // float4 outputs per head
    for (int idx = tid; idx < g * kVec; idx += nthreads) {
        const int head = idx / kVec, d4 = idx - head * kVec;
        const float LSE = s_lse[head];
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        if (LSE != -INFINITY) {
#pragma unroll 4
            for (int s = 0; s < nseg; ++s) {
                if (maybe_empty && run_is_empty(rr.i0 + s, N, P)) continue;
                const size_t r = (slot0 + s) * g + head;
                const float w = ex2((__ldcg(seg_lse + r) - LSE) * kLog2eF);
                const float4 o = __ldcg(reinterpret_cast<const float4 *>(seg_out + r * D) + d4);
                acc.x = fmaf(w, o.x, acc.x);
                acc.y = fmaf(w, o.y, acc.y);
                acc.z = fmaf(w, o.z, acc.z);
                acc.w = fmaf(w, o.w, acc.w);
            }
        }
        reinterpret_cast<float4 *>(out_row + head * D)[d4] = acc;
        if (d4 == 0) lse_row[head] = LSE;
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
