// fd_partition.cuh -- where the split stage cuts the key/value stream.
//
// "Flash-Decoding for long-context inference", section "A faster attention
// for decoding: Flash-Decoding": the keys/values are split into chunks along
// the sequence and the chunks are processed in parallel. Here every row
// (sequence b, kv head j; row index u = b*Hkv + j) contributes
// n_b = ceil(L_b / 64) tiles of 64 tokens, the rows are laid end to end in
// the order u = 0, 1, ..., and the resulting stream of N tiles is cut into P
// runs of equal length (+-1 tile): run i covers flat tiles
// [floor(i*N/P), floor((i+1)*N/P)). One run is one thread block, so every SM
// streams the same number of bytes whatever the mix of row lengths.
//
// A run that covers only part of row u writes that part (one "segment") to
// workspace slot i + u. Slots are unique: if run i ends in row u_end, run
// i + 1 starts in a row >= u_end, so its first slot is >= i + 1 + u_end.
// At most P + U - 1 slots exist.
//
// Shared by host code (fd_segments, workspace sizing) and device code.
#pragma once

#include <stdint.h>

namespace fd {

// Sticky per-device error word (FD_ERR_TIMEOUT when a wait gave up,
// FD_ERR_BOUNDS when a debug build's bounds check failed).
__device__ int g_fd_error_word;

// Debug builds (-DFD_DEBUG) check the global accesses whose indices come
// from the partition arithmetic; a failed check records FD_ERR_BOUNDS and
// the access is skipped. Release builds compile the checks away.
__device__ __forceinline__ bool debug_check(bool ok) {
    if (!ok) atomicExch(&g_fd_error_word, -13 /* FD_ERR_BOUNDS */);
    return ok;
}
#ifdef FD_DEBUG
#define FD_DCHECK(cond) ::fd::debug_check(cond)
#else
#define FD_DCHECK(cond) true
#endif


constexpr int kTileTokens = 64;

__host__ __device__ __forceinline__ int clamp_len(int L, int Lmax) {
    return L < 0 ? 0 : (L > Lmax ? Lmax : L);
}

__host__ __device__ __forceinline__ int tiles_of(int L) { return (L + kTileTokens - 1) / kTileTokens; }

// First flat tile of run i (i in [0, P]).
__host__ __device__ __forceinline__ long long run_begin(long long i, long long N, long long P) {
    return i * N / P;
}

// The run that holds flat tile t (0 <= t < N): the largest i with
// floor(i*N/P) <= t, i.e. i*N < (t+1)*P.
__host__ __device__ __forceinline__ int run_of_tile(long long t, long long N, long long P) {
    return static_cast<int>(((t + 1) * P - 1) / N);
}

}  // namespace fd
