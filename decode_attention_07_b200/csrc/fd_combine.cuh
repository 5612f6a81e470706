// fd_combine.cuh -- the final reduction over splits as a kernel of its own
// (fd_combine): one block per (sequence, kv head) row merges the segments
// that fd_split wrote, with the same merge code as the split kernel's fused
// form (fd_merge.cuh). Rows held whole by one split are left alone; rows
// with no tokens get out = 0, lse = -inf.
#pragma once

#include "fd_merge.cuh"
#include "fd_partition.cuh"
#include "fd_ptx.cuh"

namespace fd {

constexpr int kCombineThreads = 128;

struct CombineParams {
    const int32_t *seqlens;
    float *out, *lse;
    const float *seg_out, *seg_lse;
    int B, Hq, Hkv, g, Lmax, P;
};

template <int D>
__global__ void __launch_bounds__(kCombineThreads) fd_combine_kernel(const CombineParams p) {
    const long long u = blockIdx.x;
    const int b = static_cast<int>(u / p.Hkv), h = static_cast<int>(u % p.Hkv);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

    // tiles before sequence b, and in total (inputs only: safe before the wait)
    long long before = 0, total = 0;
    for (int bb = tid; bb < p.B; bb += kCombineThreads) {
        const int n = tiles_of(clamp_len(__ldg(p.seqlens + bb), p.Lmax));
        total += n;
        if (bb < b) before += n;
    }
    for (int s = 16; s > 0; s >>= 1) {
        before += __shfl_xor_sync(0xffffffffu, before, s);
        total += __shfl_xor_sync(0xffffffffu, total, s);
    }
    __shared__ long long red[2][kCombineThreads / 32];
    if (lane == 0) {
        red[0][warp] = before;
        red[1][warp] = total;
    }
    __syncthreads();
    before = total = 0;
#pragma unroll
    for (int w = 0; w < kCombineThreads / 32; ++w) {
        before += red[0][w];
        total += red[1][w];
    }
    const int n_b = tiles_of(clamp_len(__ldg(p.seqlens + b), p.Lmax));
    const size_t row0 = static_cast<size_t>(b) * p.Hq + static_cast<size_t>(h) * p.g;

    // Everything below reads what the split grid wrote, or writes next to it.
    grid_dependency_wait();
    if (!FD_DCHECK(row0 + p.g <= static_cast<size_t>(p.B) * p.Hq)) return;

    if (n_b == 0) {
        write_empty_row<D>(p.out + row0 * D, p.lse + row0, p.g, tid, kCombineThreads);
        return;
    }
    const long long N = total * p.Hkv;
    const long long first = before * p.Hkv + static_cast<long long>(h) * n_b;
    const RowRuns rr = row_runs(first, n_b, N, p.P);
    if (rr.i0 == rr.i1) return;   // one segment: the split stage wrote this row
    if (!FD_DCHECK(static_cast<size_t>(rr.i1) + static_cast<size_t>(u) <
                   static_cast<size_t>(p.P) + static_cast<size_t>(p.B) * p.Hkv - 1))
        return;
    merge_row<D>(p.seg_out, p.seg_lse, p.g, u, rr, N, p.P, p.out + row0 * D, p.lse + row0, tid, kCombineThreads);
}

}  // namespace fd
