// fd_partials.cuh -- the final reduction over partial attention results that
// were computed elsewhere: one partial (O_r, lse_r) per part r of each row,
// e.g. one per GPU when a long sequence is sharded along its tokens
// (context parallelism, as in the DISTFLASHATTN abstract on the "Related
// papers: Glinthawk" page, which distributes attention over GPUs along the
// sequence). The reduction is the one of "Flash-Decoding for long-context
// inference", section "A faster attention for decoding: Flash-Decoding":
//     LSE = M + log sum_r exp(lse_r - M),   M = max_r lse_r
//     out = sum_r exp(lse_r - LSE) * O_r    (r in increasing order)
// Parts with lse_r = -inf (no tokens) weigh nothing; a row whose every part
// is empty gets out = 0, lse = -inf.
#pragma once

#include "fd_ptx.cuh"

namespace fd {

constexpr int kPartialsThreads = 256;
constexpr float kPartialsLog2e = 1.44269504088896341f;
constexpr float kPartialsLn2 = 0.693147180559945309f;

// One thread per float4 of the output: rows x (D / 4) items. A single pass
// over the parts in order, with a running maximum (the partials are read
// once each, deterministically in part order).
__global__ void __launch_bounds__(kPartialsThreads)
    fd_merge_partials_kernel(const float *part_out, const float *part_lse, int R, long long rows, int D,
                             float *out, float *lse) {
    const int vec = D / 4;
    const long long idx = static_cast<long long>(blockIdx.x) * kPartialsThreads + threadIdx.x;
    if (idx >= rows * vec) return;
    const long long row = idx / vec;
    const int d4 = static_cast<int>(idx - row * vec);
    float M = -INFINITY, S = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int r = 0; r < R; ++r) {
        const long long pr = static_cast<long long>(r) * rows + row;
        const float ls = __ldg(part_lse + pr);
        if (ls == -INFINITY) continue;
        const float4 o = __ldg(reinterpret_cast<const float4 *>(part_out + pr * D) + d4);
        if (ls > M) {   // new maximum: rescale what has been summed so far
            const float c = ex2((M - ls) * kPartialsLog2e);
            S *= c;
            acc.x *= c;
            acc.y *= c;
            acc.z *= c;
            acc.w *= c;
            M = ls;
        }
        const float w = ex2((ls - M) * kPartialsLog2e);
        S += w;
        acc.x = fmaf(w, o.x, acc.x);
        acc.y = fmaf(w, o.y, acc.y);
        acc.z = fmaf(w, o.z, acc.z);
        acc.w = fmaf(w, o.w, acc.w);
    }
    float4 res = make_float4(0.f, 0.f, 0.f, 0.f);
    float l = -INFINITY;
    if (M != -INFINITY) {
        const float inv = 1.f / S;
        res = make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
        l = M + lg2(S) * kPartialsLn2;
    }
    reinterpret_cast<float4 *>(out + row * D)[d4] = res;
    if (d4 == 0) lse[row] = l;
}

}  // namespace fd
