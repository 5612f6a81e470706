// fd_combine.cuh -- the final reduction over splits.
//
// "Flash-Decoding for long-context inference", section "A faster attention
// for decoding: Flash-Decoding": the actual output is obtained by reducing
// over all splits, each split's contribution scaled through its
// log-sum-exp. For one row with segments s = 0..S-1 (normalised outputs O_s,
// natural-log log-sum-exps lse_s):
//     LSE = log sum_s exp(lse_s)           (max-shifted)
//     out = sum_s exp(lse_s - LSE) * O_s   (fixed order s = 0, 1, ...)
// One block per (sequence, kv head) row handles its g query heads. Rows the
// split stage wrote whole are left alone; rows with no tokens get 0 / -inf.
#pragma once

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
    const int u = blockIdx.x;
    const int b = u / p.Hkv, h = u - b * p.Hkv;
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
    __shared__ float s_lse[16];
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

    if (n_b == 0) {
        for (int idx = tid; idx < p.g * D; idx += kCombineThreads) {
            p.out[row0 * D + idx] = 0.f;
            if (idx % D == 0) p.lse[row0 + idx / D] = -INFINITY;
        }
        return;
    }
    const long long N = total * p.Hkv;
    const long long first = before * p.Hkv + static_cast<long long>(h) * n_b;
    const int i0 = run_of_tile(first, N, p.P);
    const int i1 = run_of_tile(first + n_b - 1, N, p.P);
    if (i0 == i1) return;   // one segment: the split stage wrote this row
    const int nseg = i1 - i0 + 1;
    const size_t slot0 = static_cast<size_t>(i0) + u;

    // per head: LSE over the segments (one warp per head)
    for (int head = warp; head < p.g; head += kCombineThreads / 32) {
        float mx = -INFINITY;
        for (int s = lane; s < nseg; s += 32) mx = fmaxf(mx, p.seg_lse[(slot0 + s) * p.g + head]);
        for (int sh = 16; sh > 0; sh >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, sh));
        float sum = 0.f;
        if (mx != -INFINITY)
            for (int s = lane; s < nseg; s += 32) sum += expf(p.seg_lse[(slot0 + s) * p.g + head] - mx);
        for (int sh = 16; sh > 0; sh >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, sh);
        if (lane == 0) s_lse[head] = mx == -INFINITY ? -INFINITY : mx + logf(sum);
    }
    __syncthreads();

    for (int idx = tid; idx < p.g * D; idx += kCombineThreads) {
        const int head = idx / D, d = idx - head * D;
        const float LSE = s_lse[head];
        float acc = 0.f;
        if (LSE != -INFINITY) {
            for (int s = 0; s < nseg; ++s) {
                const size_t r = (slot0 + s) * p.g + head;
                const float ls = p.seg_lse[r];
                if (ls != -INFINITY) acc += expf(ls - LSE) * p.seg_out[r * D + d];
            }
        }
        p.out[(row0 + head) * D + d] = acc;
        if (d == 0) p.lse[row0 + head] = LSE;
    }
}

}  // namespace fd
