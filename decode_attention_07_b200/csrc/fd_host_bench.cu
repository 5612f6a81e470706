// fd_host_bench.cu -- host time of one decode call through the C ABI, measured
// from C++ with nothing but the library between the caller and the driver
// (no Python, no ctypes). A decode loop on the host pays this per call to
// enqueue the kernel; the GPU time of the call is separate.
//
//   fd_host_bench B Hq Hkv D L CALLS
//
// Allocates the caches (zeros: the values do not change the host path), then
// times CALLS back-to-back calls of each entry point on one stream (enqueue
// only; the stream is synchronised after the timed loop) and prints one JSON
// object with microseconds per call. An empty kernel's launch is timed the
// same way as the floor any launch pays.
#include <cuda_runtime.h>

#include <chrono>
#include <cstdio>
#include <cstdlib>
#include <vector>

#include "fd.h"

namespace {

__global__ void empty_kernel() {}

template <class F>
double us_per_call(int calls, cudaStream_t st, F &&fn, int *rc) {
    const auto t0 = std::chrono::steady_clock::now();
    for (int i = 0; i < calls; ++i) {
        const int r = fn();
        if (r != 0 && *rc == 0) *rc = r;
    }
    const auto t1 = std::chrono::steady_clock::now();
    cudaStreamSynchronize(st);
    return std::chrono::duration<double, std::micro>(t1 - t0).count() / calls;
}

}  // namespace

int main(int argc, char **argv) {
    if (argc != 7) {
        std::fprintf(stderr, "usage: %s B Hq Hkv D L CALLS\n", argv[0]);
        return 2;
    }
    const int B = std::atoi(argv[1]), Hq = std::atoi(argv[2]), Hkv = std::atoi(argv[3]), D = std::atoi(argv[4]);
    const int L = std::atoi(argv[5]), calls = std::atoi(argv[6]);
    if (B < 1 || Hq < 1 || Hkv < 1 || L < 1 || calls < 1) return 2;
    const size_t nq = static_cast<size_t>(B) * Hq * D, nkv = static_cast<size_t>(B) * Hkv * L * D;
    uint16_t *q = nullptr, *k = nullptr, *v = nullptr;
    int32_t *seqlens = nullptr;
    float *out = nullptr, *lse = nullptr;
    void *ws = nullptr;
    const int S = fd_plan(B, Hq, Hkv, D, L);
    if (S < 1) {
        std::fprintf(stderr, "fd_plan: %s\n", fd_strerror(S));
        return 1;
    }
    const size_t wbytes = fd_workspace_bytes(B, Hq, Hkv, D, L, S);
    if (cudaMalloc(&q, nq * 2) != cudaSuccess || cudaMalloc(&k, nkv * 2) != cudaSuccess ||
        cudaMalloc(&v, nkv * 2) != cudaSuccess || cudaMalloc(&seqlens, B * 4) != cudaSuccess ||
        cudaMalloc(&out, nq * 4) != cudaSuccess || cudaMalloc(&lse, static_cast<size_t>(B) * Hq * 4) != cudaSuccess ||
        cudaMalloc(&ws, wbytes > 16 ? wbytes : 16) != cudaSuccess) {
        std::fprintf(stderr, "cudaMalloc failed\n");
        return 1;
    }
    cudaMemset(q, 0, nq * 2);
    cudaMemset(k, 0, nkv * 2);
    cudaMemset(v, 0, nkv * 2);
    std::vector<int32_t> lens(B, L);
    cudaMemcpy(seqlens, lens.data(), B * 4, cudaMemcpyHostToDevice);
    cudaStream_t st;
    cudaStreamCreateWithFlags(&st, cudaStreamNonBlocking);
    int rc = fd_workspace_init(ws, wbytes, st);
    const float scale = 0.08838834764831845f;
    auto decode = [&] { return fd_decode(B, Hq, Hkv, D, L, q, k, v, seqlens, scale, out, lse, ws, wbytes, st); };
    auto decode_s = [&] {
        return fd_decode_splits(B, Hq, Hkv, D, L, q, k, v, seqlens, scale, out, lse, ws, wbytes, S, st);
    };
    auto plan = [&] { return fd_plan(B, Hq, Hkv, D, L) > 0 ? 0 : -1; };
    auto empty = [&] {
        empty_kernel<<<1, 32, 0, st>>>();
        return cudaGetLastError() == cudaSuccess ? 0 : -1;
    };
    for (int i = 0; i < 10; ++i) {
        const int r = decode();
        if (r != 0 && rc == 0) rc = r;
        empty();
    }
    cudaStreamSynchronize(st);
    const double t_decode = us_per_call(calls, st, decode, &rc);
    const double t_splits = us_per_call(calls, st, decode_s, &rc);
    const double t_plan = us_per_call(calls, st, plan, &rc);
    const double t_empty = us_per_call(calls, st, empty, &rc);
    const int status = fd_device_status(st);
    std::printf(
        "{\"host_us_per_call\": {\"fd_decode\": %.3f, \"fd_decode_splits\": %.3f, \"fd_plan\": %.3f, "
        "\"empty_kernel_launch\": %.3f}, \"calls\": %d, \"shape\": [%d, %d, %d, %d, %d], \"num_splits\": %d, "
        "\"rc\": %d, \"status\": %d}\n",
        t_decode, t_splits, t_plan, t_empty, calls, B, Hq, Hkv, D, L, S, rc, status);
    cudaStreamDestroy(st);
    cudaFree(q);
    cudaFree(k);
    cudaFree(v);
    cudaFree(seqlens);
    cudaFree(out);
    cudaFree(lse);
    cudaFree(ws);
    return rc == 0 && status == 0 ? 0 : 1;
}
