// fd_probe.cu -- a plain HBM read-bandwidth probe: the ceiling the decode
// kernels' K/V streaming is compared against (a copy measures reads and
// writes together; decode only reads). Not part of the attention path.
//
// It streams the way the split kernel does, without the attention: one
// block per SM, one thread issuing 32 KiB bulk copies (cp.async.bulk, the
// TMA engine) into a 4-stage shared-memory ring, 128 KiB in flight per SM,
// with mbarrier completion. Chunks go to blocks round-robin. One word of
// every chunk is folded into *sink so the copies cannot be dropped.
#include <cuda_runtime.h>
#include <stdint.h>

#include "fd.h"

namespace {

constexpr int kProbeStages = 4;
constexpr uint32_t kProbeChunk = 32768;
constexpr int kProbeSmem = kProbeStages * kProbeChunk + 128;
constexpr uint64_t kProbeWaitNs = 2000000000ull;   // a bounded wait gives up after 2 s

__device__ __forceinline__ uint32_t saddr(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t now_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Wait for phase `parity` of the barrier; false after kProbeWaitNs.
__device__ __forceinline__ bool wait_phase(uint64_t *bar, uint32_t parity) {
    const uint64_t t0 = now_ns();
    while (true) {
        uint32_t ok;
        asm volatile(
            "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(ok)
            : "r"(saddr(bar)), "r"(parity)
            : "memory");
        if (ok) return true;
        if (now_ns() - t0 > kProbeWaitNs) return false;
    }
}

__device__ __forceinline__ void load_chunk(uint8_t *dst, const uint8_t *src, uint32_t bytes, uint64_t *bar) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(saddr(bar)), "r"(bytes)
                 : "memory");
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     saddr(dst)),
                 "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(saddr(bar))
                 : "memory");
}

__global__ void __launch_bounds__(32, 1) fd_read_probe_kernel(const uint8_t *buf, size_t bytes,
                                                              unsigned long long *sink, int *timed_out) {
    extern __shared__ __align__(128) uint8_t smem[];
    uint64_t *bar = reinterpret_cast<uint64_t *>(smem + kProbeStages * kProbeChunk);
    if (threadIdx.x != 0) return;
    const size_t nchunks = (bytes + kProbeChunk - 1) / kProbeChunk;
    const size_t mine = blockIdx.x < nchunks ? (nchunks - blockIdx.x + gridDim.x - 1) / gridDim.x : 0;
    if (mine == 0) return;
    for (int s = 0; s < kProbeStages; ++s)
        asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(saddr(&bar[s])) : "memory");
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    auto chunk_at = [&](size_t k, uint32_t *len) {   // this block's k-th chunk
        const size_t c = blockIdx.x + k * gridDim.x;
        const size_t off = c * kProbeChunk;
        *len = static_cast<uint32_t>(bytes - off < kProbeChunk ? bytes - off : kProbeChunk);
        return buf + off;
    };
    for (size_t k = 0; k < mine && k < kProbeStages; ++k) {
        uint32_t len;
        const uint8_t *src = chunk_at(k, &len);
        load_chunk(smem + k * kProbeChunk, src, len, &bar[k]);
    }
    uint32_t acc = 0;
    for (size_t k = 0; k < mine; ++k) {
        const int s = static_cast<int>(k % kProbeStages);
        if (!wait_phase(&bar[s], static_cast<uint32_t>((k / kProbeStages) & 1))) {
            // give up, but leave only once the copies already issued have landed,
            // chunk k's own included (each of those waits bounded too)
            atomicExch(timed_out, 1);
            wait_phase(&bar[s], static_cast<uint32_t>((k / kProbeStages) & 1));
            for (size_t j = k + 1; j < mine && j < k + kProbeStages; ++j)
                wait_phase(&bar[j % kProbeStages], static_cast<uint32_t>((j / kProbeStages) & 1));
            return;
        }
        acc ^= *reinterpret_cast<volatile uint32_t *>(smem + s * kProbeChunk);
        if (k + kProbeStages < mine) {
            uint32_t len;
            const uint8_t *src = chunk_at(k + kProbeStages, &len);
            load_chunk(smem + s * kProbeChunk, src, len, &bar[s]);
        }
    }
    atomicXor(sink, static_cast<unsigned long long>(acc));
}

}  // namespace

extern "C" int fd_read_probe(const void *buf, size_t bytes, unsigned long long *sink, void *stream) {
    if (bytes == 0) return FD_OK;
    if (!buf || !sink) return FD_ERR_NULL_POINTER;
    if (reinterpret_cast<uintptr_t>(buf) % 16 != 0 || bytes % 16 != 0 || reinterpret_cast<uintptr_t>(sink) % 8 != 0)
        return FD_ERR_ALIGNMENT;
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) !=
                                                  cudaSuccess) {
        cudaGetLastError();
        return FD_ERR_DEVICE;
    }
    if (cudaFuncSetAttribute(fd_read_probe_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kProbeSmem) !=
        cudaSuccess) {
        cudaGetLastError();
        return FD_ERR_LAUNCH;
    }
    // the flag of a bounded wait that gave up: the word after *sink's 8 bytes is not ours,
    // so it lives in the sink's upper half: the probe never sets bits 32..62 otherwise
    int *timed_out = reinterpret_cast<int *>(sink) + 1;
    fd_read_probe_kernel<<<sms, 32, kProbeSmem, static_cast<cudaStream_t>(stream)>>>(
        static_cast<const uint8_t *>(buf), bytes, sink, timed_out);
    if (cudaGetLastError() != cudaSuccess) return FD_ERR_LAUNCH;
    return FD_OK;
}
