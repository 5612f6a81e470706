// fd_api.cu -- the C ABI declared in include/fd.h: argument checks, the
// split planner, tensor-map encoding and the two launches.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "fd.h"
#include "fd_combine.cuh"
#include "fd_partials.cuh"
#include "fd_partition.cuh"
#include "fd_quant.cuh"
#include "fd_split.cuh"

namespace {

constexpr int kVersion = 100;               // 0.1.0
constexpr int kMinTilesPerSplit = 4;        // a split streams at least 256 tokens per kv head
constexpr int kMidTilesPerSm = 16;          // up to this many tiles per SM, splits come in multiples of 32
constexpr int kMaxDevices = 64;
constexpr float kLog2e = 1.4426950408889634f;

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// ----------------------------------------------------------- shape checks --
int check_shape(int B, int Hq, int Hkv, int D, int max_len) {
    if (B < 1 || Hq < 1 || Hkv < 1 || max_len < 0) return FD_ERR_SHAPE;
    if (Hq % Hkv != 0 || Hq / Hkv > FD_MAX_GROUP) return FD_ERR_GROUP;
    if (D != 64 && D != 128) return FD_ERR_HEAD_DIM;
    // sizes kept inside 32-bit grid/tensor-map dimensions and 64-bit run arithmetic
    const long long rows = static_cast<long long>(B) * Hkv;
    if (rows > 0x7fffffffLL || static_cast<long long>(B) * Hq > 0x7fffffffLL) return FD_ERR_SHAPE;
    const long long tiles = rows * fd::tiles_of(max_len);
    if (tiles > (1LL << 44)) return FD_ERR_SHAPE;
    return FD_OK;
}

long long num_slots(int B, int Hkv, int num_splits) {
    return static_cast<long long>(num_splits) + static_cast<long long>(B) * Hkv - 1;
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Workspace: seg_out [slots][g][D] fp32 | seg_lse [slots][g] fp32 | row tickets [B*Hkv] int32
// followed by chunk tickets [slots] int32,
// each part 256-byte aligned.
struct WorkspaceLayout {
    size_t seg_out, seg_lse, tickets, total;
};

WorkspaceLayout workspace_layout(int B, int Hq, int Hkv, int D, int num_splits) {
    WorkspaceLayout w{0, 0, 0, 0};
    if (num_splits <= 1) return w;
    const size_t slots = static_cast<size_t>(num_slots(B, Hkv, num_splits));
    const size_t g = static_cast<size_t>(Hq / Hkv);
    w.seg_out = 0;
    w.seg_lse = align256(slots * g * D * sizeof(float));
    w.tickets = w.seg_lse + align256(slots * g * sizeof(float));
    w.total = w.tickets + align256((static_cast<size_t>(B) * Hkv + slots) * sizeof(int));
    return w;
}

size_t workspace_bytes(int B, int Hq, int Hkv, int D, int num_splits) {
    return workspace_layout(B, Hq, Hkv, D, num_splits).total;
}

// ------------------------------------------------------------ device info --
struct DeviceInfo {
    bool queried = false;
    int status = FD_OK;
    int sms = 0;
};
DeviceInfo g_devices[kMaxDevices];
std::mutex g_mutex;

int current_device(int *dev) {
    if (cudaGetDevice(dev) != cudaSuccess) {
        cudaGetLastError();
        return FD_ERR_DEVICE;
    }
    if (*dev < 0 || *dev >= kMaxDevices) return FD_ERR_DEVICE;
    return FD_OK;
}

int device_sms(int *sms) {
    int dev;
    int rc = current_device(&dev);
    if (rc != FD_OK) return rc;
    std::lock_guard<std::mutex> lock(g_mutex);
    DeviceInfo &d = g_devices[dev];
    if (!d.queried) {
        int major = 0, minor = 0, n = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
            cudaGetLastError();
            d.status = FD_ERR_DEVICE;
        } else if (major != 10 || minor != 0) {
            d.status = FD_ERR_DEVICE;   // built for sm_100a only
        } else {
            d.status = FD_OK;
            d.sms = n;
        }
        d.queried = true;
    }
    *sms = d.sms;
    return d.status;
}

// ------------------------------------------------------------ tensor maps --
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
        else
            cudaGetLastError();
    });
    return fn;
}

// Encoded tensor maps, cached per device. A map holds only the base address,
// the shape, the strides and the box, so a map encoded once for a buffer
// stays valid for every later call on that buffer (and for a new buffer
// that happens to reuse the address with the same shape). A decode loop that
// reuses its caches thus encodes each map once instead of once per call.
// Entries are replaced round-robin when the cache is full.
struct MapKey {
    int dtype, rank, swizzle;
    const void *base;
    cuuint64_t dims[5], strides[4];
    cuuint32_t box[5];
};
struct MapEntry {
    MapKey key;
    CUtensorMap map;
};
constexpr int kMapCacheEntries = 32;
struct MapCache {
    MapEntry e[kMapCacheEntries];
    int size = 0, next = 0;
};
MapCache g_map_cache[kMaxDevices];
std::mutex g_map_mutex;

// cuTensorMapEncodeTiled with element strides 1, no interleave, 256-byte L2
// promotion and no fill, through the cache.
int encode_tiled(CUtensorMap *map, CUtensorMapDataType dtype, int rank, const void *base, const cuuint64_t *dims,
                 const cuuint64_t *strides, const cuuint32_t *box, CUtensorMapSwizzle swz) {
    int dev;
    if (current_device(&dev) != FD_OK) return FD_ERR_DEVICE;
    MapKey k;
    std::memset(&k, 0, sizeof k);   // padding included: keys are compared bytewise
    k.dtype = static_cast<int>(dtype);
    k.rank = rank;
    k.swizzle = static_cast<int>(swz);
    k.base = base;
    for (int i = 0; i < rank; ++i) {
        k.dims[i] = dims[i];
        k.box[i] = box[i];
        if (i + 1 < rank) k.strides[i] = strides[i];
    }
    {
        std::lock_guard<std::mutex> lock(g_map_mutex);
        MapCache &c = g_map_cache[dev];
        for (int i = 0; i < c.size; ++i)
            if (std::memcmp(&c.e[i].key, &k, sizeof k) == 0) {
                *map = c.e[i].map;
                return FD_OK;
            }
    }
    auto fn = encode_fn();
    if (!fn) return FD_ERR_LAUNCH;
    cuuint32_t estr[5] = {1, 1, 1, 1, 1};
    const CUresult r = fn(map, dtype, static_cast<cuuint32_t>(rank), const_cast<void *>(base), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return FD_ERR_LAUNCH;
    std::lock_guard<std::mutex> lock(g_map_mutex);
    MapCache &c = g_map_cache[dev];
    const int slot = c.size < kMapCacheEntries ? c.size++ : (c.next++ % kMapCacheEntries);
    c.e[slot].key = k;
    c.e[slot].map = *map;
    return FD_OK;
}

// K or V cache [B*Hkv rows][Lmax][D] as a 3-D tensor (D innermost). bf16:
// box = 64 head-dim elements (128 bytes, 128-byte swizzle) x 64 tokens x 1
// row. 8-bit codes (one_byte): box = all D codes of a token (128 bytes with
// the 128-byte swizzle for D = 128, 64 bytes with the 64-byte one for D = 64).
int encode_cache_map(CUtensorMap *map, const void *base, int D, int Lmax, long long rows, bool one_byte = false) {
    const cuuint64_t e = one_byte ? 1 : 2;
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(Lmax), static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * e, static_cast<cuuint64_t>(Lmax) * D * e};
    cuuint32_t box[3] = {one_byte ? static_cast<cuuint32_t>(D) : 64u, static_cast<cuuint32_t>(fd::kTileTokens), 1};
    const CUtensorMapSwizzle swz = one_byte && D == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B;
    return encode_tiled(map, one_byte ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, base, dims,
                        strides, box, swz);
}

// bf16 cache at D = 128 for the one-head consumer: each 256-byte token row
// seen as two 128-byte halves, {64 elements, 2 halves, Lmax tokens, rows},
// box {64, 2, 64, 1}: one copy brings a whole 64-token tile of one row as
// [token][half][128 B] with the 128-byte swizzle.
int encode_cache_map_rows(CUtensorMap *map, const void *base, int Lmax, long long rows) {
    cuuint64_t dims[4] = {64, 2, static_cast<cuuint64_t>(Lmax), static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[3] = {128, 256, static_cast<cuuint64_t>(Lmax) * 256};
    cuuint32_t box[4] = {64, 2, static_cast<cuuint32_t>(fd::kTileTokens), 1};
    return encode_tiled(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, base, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
}

// Paged K or V pool as a 3-D tensor, head-dim innermost. Head-major pages
// [num_pages][Hkv][page_size][D]: the token rows of one (page, head) are
// contiguous, so {D, page_size, num_pages * Hkv}, box {64, rows, 1}, row
// z = page * Hkv + head. Token-major pages [num_pages][page_size][Hkv][D]:
// page and token merge into one dimension, {D, Hkv, num_pages * page_size},
// box {64, 1, rows}, z = page * page_size + token. rows = min(page_size, 64);
// 128-byte swizzle as above. A page index outside the pool falls outside the
// tensor either way (TMA fills zeros). 8-bit codes (one_byte): boxes of all D
// codes of a token (64-byte swizzle for D = 64).
int encode_paged_map(CUtensorMap *map, const void *base, int D, int page_size, int Hkv, long long num_pages,
                     bool nhd, bool one_byte = false) {
    const cuuint64_t e = one_byte ? 1 : 2;   // 8-bit codes or bf16
    const cuuint32_t rows = static_cast<cuuint32_t>(page_size < fd::kTileTokens ? page_size : fd::kTileTokens);
    const cuuint64_t row = static_cast<cuuint64_t>(D) * e;   // bytes of one token of one head
    cuuint64_t dims[3], strides[2];
    cuuint32_t box[3];
    dims[0] = static_cast<cuuint64_t>(D);
    box[0] = one_byte ? static_cast<cuuint32_t>(D) : 64u;
    if (nhd) {
        dims[1] = static_cast<cuuint64_t>(Hkv);
        dims[2] = static_cast<cuuint64_t>(num_pages) * page_size;
        strides[0] = row;
        strides[1] = static_cast<cuuint64_t>(Hkv) * row;
        box[1] = 1;
        box[2] = rows;
    } else {
        dims[1] = static_cast<cuuint64_t>(page_size);
        dims[2] = static_cast<cuuint64_t>(num_pages) * Hkv;
        strides[0] = row;
        strides[1] = static_cast<cuuint64_t>(page_size) * row;
        box[1] = rows;
        box[2] = 1;
    }
    const CUtensorMapSwizzle swz = one_byte && D == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B;
    return encode_tiled(map, one_byte ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, base, dims,
                        strides, box, swz);
}

// Small pages at D = 128 (page_size < 64): each 256-byte token row viewed as
// two 128-byte halves, so one box brings a whole page of one kv head,
// [token][half][128 B] with the 128-byte swizzle. Head-major pages:
// {64, 2, page_size, Hkv, num_pages}, box {64, 2, page_size, 1, 1}; token-major:
// {64, 2, Hkv, page_size, num_pages}, box {64, 2, 1, page_size, 1}.
int encode_paged_map_rows(CUtensorMap *map, const void *base, int page_size, int Hkv, long long num_pages, bool nhd,
                          int pages_per_box = 1) {
    const cuuint64_t row = 256;   // bytes of one token of one head (D = 128, bf16)
    cuuint64_t dims[5], strides[4];
    cuuint32_t box[5];
    dims[0] = 64;
    dims[1] = 2;
    dims[4] = static_cast<cuuint64_t>(num_pages);
    strides[0] = 128;
    box[0] = 64;
    box[1] = 2;
    box[4] = static_cast<cuuint32_t>(pages_per_box);
    if (nhd) {
        dims[2] = static_cast<cuuint64_t>(Hkv);
        dims[3] = static_cast<cuuint64_t>(page_size);
        strides[1] = row;
        strides[2] = static_cast<cuuint64_t>(Hkv) * row;
        box[2] = 1;
        box[3] = static_cast<cuuint32_t>(page_size);
    } else {
        dims[2] = static_cast<cuuint64_t>(page_size);
        dims[3] = static_cast<cuuint64_t>(Hkv);
        strides[1] = row;
        strides[2] = static_cast<cuuint64_t>(page_size) * row;
        box[2] = static_cast<cuuint32_t>(page_size);
        box[3] = 1;
    }
    strides[3] = static_cast<cuuint64_t>(page_size) * Hkv * row;
    return encode_tiled(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, base, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
}

// Small pages (page_size < 64): one box over a run of 64 / page_size
// consecutive pages of one kv head, for tiles whose pages are consecutive in
// the pool (the same bytes at the same places as one box per page). Head-major
// pages: {D, page_size, Hkv, num_pages}, box {cols, page_size, 1, pages};
// token-major: {D, Hkv, num_pages * page_size}, box {cols, 1, 64} (the pages'
// tokens are one range of the third dimension). cols = 64 bf16 or all D codes.
int encode_paged_run_map(CUtensorMap *map, const void *base, int D, int page_size, int Hkv, long long num_pages,
                         bool nhd, bool one_byte) {
    const cuuint64_t e = one_byte ? 1 : 2;
    const cuuint64_t row = static_cast<cuuint64_t>(D) * e;
    const cuuint32_t cols = one_byte ? static_cast<cuuint32_t>(D) : 64u;
    const CUtensorMapSwizzle swz = one_byte && D == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B;
    const CUtensorMapDataType dt = one_byte ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    if (nhd) {
        cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(Hkv),
                              static_cast<cuuint64_t>(num_pages) * page_size};
        cuuint64_t strides[2] = {row, static_cast<cuuint64_t>(Hkv) * row};
        cuuint32_t box[3] = {cols, 1, static_cast<cuuint32_t>(fd::kTileTokens)};
        return encode_tiled(map, dt, 3, base, dims, strides, box, swz);
    }
    cuuint64_t dims[4] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(page_size), static_cast<cuuint64_t>(Hkv),
                          static_cast<cuuint64_t>(num_pages)};
    cuuint64_t strides[3] = {row, static_cast<cuuint64_t>(page_size) * row,
                             static_cast<cuuint64_t>(page_size) * Hkv * row};
    cuuint32_t box[4] = {cols, static_cast<cuuint32_t>(page_size), 1,
                         static_cast<cuuint32_t>(fd::kTileTokens / page_size)};
    return encode_tiled(map, dt, 4, base, dims, strides, box, swz);
}

// Host-side failure injection for tests: with FD_TEST_FAIL_LAUNCH set in the
// environment (to anything but "0"), every kernel launch of the library is
// skipped and reported as FD_ERR_LAUNCH, as a failed launch would be. Read
// once per process.
bool inject_launch_failure() {
    static const bool fail = [] {
        const char *v = std::getenv("FD_TEST_FAIL_LAUNCH");
        return v != nullptr && v[0] != '\0' && !(v[0] == '0' && v[1] == '\0');
    }();
    return fail;
}

// Debug builds: FD_DEBUG_WITHHOLD=<n> makes block 0 of the split kernel arm
// the barrier of its n-th tile without issuing the copy, so a consumer's
// bounded wait runs out (tests of the timeout path). Release builds: off.
int debug_withhold() {
#ifdef FD_DEBUG
    const char *v = std::getenv("FD_DEBUG_WITHHOLD");
    return v != nullptr ? std::atoi(v) : -1;
#else
    return -1;
#endif
}

// Debug builds: FD_DEBUG_SPOIL_GUESS=1 makes the split kernel's pre-wait guess
// of each block's start wrong, to run the restart path. Release builds: off.
int debug_spoil_guess() {
#ifdef FD_DEBUG
    const char *v = std::getenv("FD_DEBUG_SPOIL_GUESS");
    return v != nullptr && v[0] == '1' ? 1 : 0;
#else
    return 0;
#endif
}

// ---------------------------------------------------------------- launches --
template <int D, class Consumer, bool kFused, bool kPaged>
int launch_split_t(const CUtensorMap &tk, const CUtensorMap &tv, const fd::SplitParams &p, cudaStream_t st,
                   const CUtensorMap *rk = nullptr, const CUtensorMap *rv = nullptr) {
    constexpr int smem = fd::SplitConfig<D, Consumer::G, Consumer::kElemBytes, kPaged>::kSmemBytes;
    auto kern = fd::fd_split_kernel<D, Consumer, kFused, kPaged>;
    // the attribute is per function and device; set it once per device
    static std::once_flag once[kMaxDevices];
    static cudaError_t attr_err[kMaxDevices];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        cudaGetLastError();
        return FD_ERR_DEVICE;
    }
    std::call_once(once[dev], [&] {
        attr_err[dev] = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    });
    if (attr_err[dev] != cudaSuccess) {
        cudaGetLastError();
        return FD_ERR_LAUNCH;
    }
    // programmatic dependent launch: the prologue overlaps the previous
    // kernel's tail; the kernel waits for it before reading any input
    cudaLaunchConfig_t cfg;
    std::memset(&cfg, 0, sizeof cfg);
    cfg.gridDim = dim3(static_cast<unsigned>(p.P));
    cfg.blockDim = dim3(fd::split_threads<kPaged>());
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (inject_launch_failure()) return FD_ERR_LAUNCH;
    // the maps of consecutive page runs (small pages only; never read otherwise)
    if (cudaLaunchKernelEx(&cfg, kern, tk, tv, rk ? *rk : tk, rv ? *rv : tv, p) != cudaSuccess) {
        cudaGetLastError();
        return FD_ERR_LAUNCH;
    }
    return FD_OK;
}

template <bool kFused, bool kPaged = false>
int launch_split(int D, int g, const CUtensorMap &tk, const CUtensorMap &tv, const fd::SplitParams &p,
                 cudaStream_t st, const CUtensorMap *rk = nullptr, const CUtensorMap *rv = nullptr) {
    if (D == 128) {
        if (g == 1) return launch_split_t<128, fd::HeadConsumer<128>, kFused, kPaged>(tk, tv, p, st, rk, rv);
        if (g <= 8) return launch_split_t<128, fd::GroupConsumer<128, 1>, kFused, kPaged>(tk, tv, p, st, rk, rv);
        return launch_split_t<128, fd::GroupConsumer<128, 2>, kFused, kPaged>(tk, tv, p, st, rk, rv);
    }
    if (g == 1) return launch_split_t<64, fd::HeadConsumer<64>, kFused, kPaged>(tk, tv, p, st, rk, rv);
    if (g <= 8) return launch_split_t<64, fd::GroupConsumer<64, 1>, kFused, kPaged>(tk, tv, p, st, rk, rv);
    return launch_split_t<64, fd::GroupConsumer<64, 2>, kFused, kPaged>(tk, tv, p, st, rk, rv);
}

// 8-bit caches: the tensor-core consumer for every column count (fused form).
template <bool kE4M3, bool kPaged = false>
int launch_split_quant(int D, int cols, const CUtensorMap &tk, const CUtensorMap &tv, const fd::SplitParams &p,
                       cudaStream_t st, const CUtensorMap *rk = nullptr, const CUtensorMap *rv = nullptr) {
    // up to 8 columns: four groups of two warps, 32 tokens per warp (more work
    // in flight per warp); 16 columns: the default two groups of four
    if (D == 128) {
        if (cols <= 8)
            return launch_split_t<128, fd::QuantConsumer<128, 1, kE4M3, 32>, true, kPaged>(tk, tv, p, st, rk, rv);
        return launch_split_t<128, fd::QuantConsumer<128, 2, kE4M3, 16>, true, kPaged>(tk, tv, p, st, rk, rv);
    }
    if (cols <= 8) return launch_split_t<64, fd::QuantConsumer<64, 1, kE4M3, 32>, true, kPaged>(tk, tv, p, st, rk, rv);
    return launch_split_t<64, fd::QuantConsumer<64, 2, kE4M3, 16>, true, kPaged>(tk, tv, p, st, rk, rv);
}

int launch_combine(int D, const fd::CombineParams &p, cudaStream_t st, bool after_split) {
    cudaLaunchConfig_t cfg;
    std::memset(&cfg, 0, sizeof cfg);
    cfg.gridDim = dim3(static_cast<unsigned>(p.B) * static_cast<unsigned>(p.Hkv));
    cfg.blockDim = dim3(fd::kCombineThreads);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = after_split ? 1 : 0;
    if (inject_launch_failure()) return FD_ERR_LAUNCH;
    cudaError_t e = D == 128 ? cudaLaunchKernelEx(&cfg, fd::fd_combine_kernel<128>, p)
                             : cudaLaunchKernelEx(&cfg, fd::fd_combine_kernel<64>, p);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return FD_ERR_LAUNCH;
    }
    return FD_OK;
}

struct Problem {
    int B, Hq, Hkv, D, max_len;
    const uint16_t *q, *k, *v;
    const int32_t *seqlens;
    float scale;
    float *out, *lse;
    void *ws;
    size_t ws_bytes;
    int num_splits;
    cudaStream_t stream;
};

// Checks shared by every compute entry point (no CUDA call).
int check_problem(const Problem &pr, bool need_kv) {
    int rc = check_shape(pr.B, pr.Hq, pr.Hkv, pr.D, pr.max_len);
    if (rc != FD_OK) return rc;
    if (pr.num_splits < 1 || pr.num_splits > FD_MAX_SPLITS) return FD_ERR_SPLITS;
    if (!pr.seqlens || !pr.out || !pr.lse) return FD_ERR_NULL_POINTER;
    // with max_len == 0 no token exists and q/k/v are never read (they may be NULL)
    const bool reads_kv = need_kv && pr.max_len > 0;
    if (reads_kv && (!pr.q || !pr.k || !pr.v)) return FD_ERR_NULL_POINTER;
    if (!aligned(pr.seqlens, 4) || !aligned(pr.out, 16) || !aligned(pr.lse, 4)) return FD_ERR_ALIGNMENT;
    if (reads_kv && (!aligned(pr.q, 16) || !aligned(pr.k, 16) || !aligned(pr.v, 16))) return FD_ERR_ALIGNMENT;
    const size_t need = workspace_bytes(pr.B, pr.Hq, pr.Hkv, pr.D, pr.num_splits);
    if (need > 0) {
        if (!pr.ws || pr.ws_bytes < need) return FD_ERR_WORKSPACE;
        if (!aligned(pr.ws, 16)) return FD_ERR_ALIGNMENT;
    }
    const long long tiles = static_cast<long long>(pr.B) * pr.Hkv * fd::tiles_of(pr.max_len);
    if (tiles > 0 && (tiles * pr.num_splits) > (1LL << 62)) return FD_ERR_SHAPE;
    return FD_OK;
}

// `q_len` query positions per sequence: a segment holds q_len * g columns.
void seg_pointers(const Problem &pr, float **so, float **sl, int **tickets, int q_len = 1) {
    const WorkspaceLayout w = workspace_layout(pr.B, pr.Hq * q_len, pr.Hkv, pr.D, pr.num_splits);
    if (w.total == 0) {
        *so = *sl = nullptr;
        *tickets = nullptr;
        return;
    }
    char *base = static_cast<char *>(pr.ws);
    *so = reinterpret_cast<float *>(base + w.seg_out);
    *sl = reinterpret_cast<float *>(base + w.seg_lse);
    *tickets = reinterpret_cast<int *>(base + w.tickets);
}

// The split kernel; `fused` adds the in-kernel combine (fd_decode), without it
// the segments are left for fd_combine. q_len > 1: several queries per
// sequence (pr.Hq counts query heads of one query position).
int run_split(const Problem &pr, bool fused, int q_len = 1) {
    int sms;
    int rc = device_sms(&sms);
    if (rc != FD_OK) return rc;
    CUtensorMap tk, tv;
    std::memset(&tk, 0, sizeof tk);
    std::memset(&tv, 0, sizeof tv);
    const long long rows = static_cast<long long>(pr.B) * pr.Hkv;
    // one head per kv head at D = 128: one copy per K or V tile (see encode_cache_map_rows)
    const bool rows_map = pr.D == 128 && pr.Hq / pr.Hkv * q_len == 1;
    if (pr.max_len > 0) {
        if (rows_map) {
            if ((rc = encode_cache_map_rows(&tk, pr.k, pr.max_len, rows)) != FD_OK) return rc;
            if ((rc = encode_cache_map_rows(&tv, pr.v, pr.max_len, rows)) != FD_OK) return rc;
        } else {
            if ((rc = encode_cache_map(&tk, pr.k, pr.D, pr.max_len, rows)) != FD_OK) return rc;
            if ((rc = encode_cache_map(&tv, pr.v, pr.D, pr.max_len, rows)) != FD_OK) return rc;
        }
    } else if (!fused) {
        return FD_OK;   // no tokens anywhere: the combine writes every row
    }
    fd::SplitParams p;
    p.q = pr.q;
    p.seqlens = pr.seqlens;
    p.out = pr.out;
    p.lse = pr.lse;
    seg_pointers(pr, &p.seg_out, &p.seg_lse, &p.row_tickets, q_len);
    p.chunk_tickets = p.row_tickets ? p.row_tickets + static_cast<size_t>(pr.B) * pr.Hkv : nullptr;
    p.B = pr.B;
    p.Hq = pr.Hq;
    p.Hkv = pr.Hkv;
    p.g = pr.Hq / pr.Hkv;
    p.Lmax = pr.max_len;
    p.P = pr.num_splits;
    p.q_len = q_len;
    p.cols = p.g * q_len;
    p.scale_log2e = pr.scale * kLog2e;
    p.block_table = nullptr;
    p.max_pages = 0;
    p.page_shift = 0;
    p.kv_nhd = 0;
    p.num_pages = 0;
    p.k_scale = p.v_scale = nullptr;
    p.k_base = pr.k;
    p.v_base = pr.v;
    p.debug_withhold = debug_withhold();
    p.debug_spoil_guess = debug_spoil_guess();
    // with max_len == 0 every block finds zero tiles and only writes empty rows;
    // the (unused) tensor maps stay zeroed
    if (rows_map)
        return fused ? launch_split_t<128, fd::HeadConsumer<128, true>, true, false>(tk, tv, p, pr.stream)
                     : launch_split_t<128, fd::HeadConsumer<128, true>, false, false>(tk, tv, p, pr.stream);
    return fused ? launch_split<true>(pr.D, p.cols, tk, tv, p, pr.stream)
                 : launch_split<false>(pr.D, p.cols, tk, tv, p, pr.stream);
}

struct PagedLayout {
    const int32_t *block_table;
    int page_size, num_pages, max_pages;
    bool nhd;
};

// Paged caches: bf16 (kv_type 0) or 8-bit codes (FD_KV_E4M3 / FD_KV_INT8 with
// per-kv-head scales), q_len queries per sequence.
int run_split_paged(const Problem &pr, const PagedLayout &pl, int q_len = 1, int kv_type = 0,
                    const float *k_scale = nullptr, const float *v_scale = nullptr) {
    int sms;
    int rc = device_sms(&sms);
    if (rc != FD_OK) return rc;
    CUtensorMap tk, tv;
    const bool quant = kv_type != 0;
    // bf16 at D = 128 with small pages: one box per page (both 128-byte halves of a row)
    const bool rows_map = !quant && pr.D == 128 && pl.page_size < fd::kTileTokens;
    // small pages: maps of runs of 64 / page_size consecutive pages (one box per such tile)
    CUtensorMap rk, rv;
    const bool small = pl.page_size < fd::kTileTokens && pl.num_pages >= fd::kTileTokens / pl.page_size;
    if (rows_map) {
        if ((rc = encode_paged_map_rows(&tk, pr.k, pl.page_size, pr.Hkv, pl.num_pages, pl.nhd)) != FD_OK) return rc;
        if ((rc = encode_paged_map_rows(&tv, pr.v, pl.page_size, pr.Hkv, pl.num_pages, pl.nhd)) != FD_OK) return rc;
        const int ppb = fd::kTileTokens / pl.page_size;
        if (small) {
            if ((rc = encode_paged_map_rows(&rk, pr.k, pl.page_size, pr.Hkv, pl.num_pages, pl.nhd, ppb)) != FD_OK)
                return rc;
            if ((rc = encode_paged_map_rows(&rv, pr.v, pl.page_size, pr.Hkv, pl.num_pages, pl.nhd, ppb)) != FD_OK)
                return rc;
        }
    } else {
        if ((rc = encode_paged_map(&tk, pr.k, pr.D, pl.page_size, pr.Hkv, pl.num_pages, pl.nhd, quant)) != FD_OK)
            return rc;
        if ((rc = encode_paged_map(&tv, pr.v, pr.D, pl.page_size, pr.Hkv, pl.num_pages, pl.nhd, quant)) != FD_OK)
            return rc;
        if (small) {
            if ((rc = encode_paged_run_map(&rk, pr.k, pr.D, pl.page_size, pr.Hkv, pl.num_pages, pl.nhd, quant)) != FD_OK)
                return rc;
            if ((rc = encode_paged_run_map(&rv, pr.v, pr.D, pl.page_size, pr.Hkv, pl.num_pages, pl.nhd, quant)) != FD_OK)
                return rc;
        }
    }
    const CUtensorMap *rkp = small ? &rk : nullptr, *rvp = small ? &rv : nullptr;
    fd::SplitParams p;
    p.q = pr.q;
    p.seqlens = pr.seqlens;
    p.out = pr.out;
    p.lse = pr.lse;
    seg_pointers(pr, &p.seg_out, &p.seg_lse, &p.row_tickets, q_len);
    p.chunk_tickets = p.row_tickets ? p.row_tickets + static_cast<size_t>(pr.B) * pr.Hkv : nullptr;
    p.B = pr.B;
    p.Hq = pr.Hq;
    p.Hkv = pr.Hkv;
    p.g = pr.Hq / pr.Hkv;
    p.Lmax = pr.max_len;
    p.P = pr.num_splits;
    p.q_len = q_len;
    p.cols = p.g * q_len;
    p.scale_log2e = pr.scale * kLog2e;
    p.block_table = pl.block_table;
    p.max_pages = pl.max_pages;
    p.page_shift = 0;
    while ((1 << p.page_shift) < pl.page_size) ++p.page_shift;
    p.kv_nhd = pl.nhd ? 1 : 0;
    p.num_pages = pl.num_pages;
    p.k_scale = k_scale;
    p.v_scale = v_scale;
    p.k_base = p.v_base = nullptr;   // paged pools: no contiguous span to prefetch
    p.debug_withhold = debug_withhold();
    p.debug_spoil_guess = debug_spoil_guess();
    if (quant)
        return kv_type == FD_KV_E4M3 ? launch_split_quant<true, true>(pr.D, p.cols, tk, tv, p, pr.stream, rkp, rvp)
                                     : launch_split_quant<false, true>(pr.D, p.cols, tk, tv, p, pr.stream, rkp, rvp);
    if (rows_map) {
        if (p.cols == 1)
            return launch_split_t<128, fd::HeadConsumer<128, true>, true, true>(tk, tv, p, pr.stream, rkp, rvp);
        if (p.cols <= 8)
            return launch_split_t<128, fd::GroupConsumer<128, 1, true>, true, true>(tk, tv, p, pr.stream, rkp, rvp);
        return launch_split_t<128, fd::GroupConsumer<128, 2, true>, true, true>(tk, tv, p, pr.stream, rkp, rvp);
    }
    return launch_split<true, true>(pr.D, p.cols, tk, tv, p, pr.stream, rkp, rvp);
}

// Fused split kernel over an 8-bit cache (pr.k / pr.v point at the codes).
int run_split_quant(const Problem &pr, int q_len, int kv_type, const float *k_scale, const float *v_scale) {
    int sms;
    int rc = device_sms(&sms);
    if (rc != FD_OK) return rc;
    CUtensorMap tk, tv;
    std::memset(&tk, 0, sizeof tk);
    std::memset(&tv, 0, sizeof tv);
    const long long rows = static_cast<long long>(pr.B) * pr.Hkv;
    if (pr.max_len > 0) {
        if ((rc = encode_cache_map(&tk, pr.k, pr.D, pr.max_len, rows, true)) != FD_OK) return rc;
        if ((rc = encode_cache_map(&tv, pr.v, pr.D, pr.max_len, rows, true)) != FD_OK) return rc;
    }
    fd::SplitParams p;
    p.q = pr.q;
    p.seqlens = pr.seqlens;
    p.out = pr.out;
    p.lse = pr.lse;
    seg_pointers(pr, &p.seg_out, &p.seg_lse, &p.row_tickets, q_len);
    p.chunk_tickets = p.row_tickets ? p.row_tickets + static_cast<size_t>(pr.B) * pr.Hkv : nullptr;
    p.B = pr.B;
    p.Hq = pr.Hq;
    p.Hkv = pr.Hkv;
    p.g = pr.Hq / pr.Hkv;
    p.Lmax = pr.max_len;
    p.P = pr.num_splits;
    p.q_len = q_len;
    p.cols = p.g * q_len;
    p.scale_log2e = pr.scale * kLog2e;
    p.block_table = nullptr;
    p.max_pages = 0;
    p.page_shift = 0;
    p.kv_nhd = 0;
    p.num_pages = 0;
    p.k_scale = k_scale;
    p.v_scale = v_scale;
    p.k_base = pr.k;
    p.v_base = pr.v;
    p.debug_withhold = debug_withhold();
    p.debug_spoil_guess = debug_spoil_guess();
    return kv_type == FD_KV_E4M3 ? launch_split_quant<true>(pr.D, p.cols, tk, tv, p, pr.stream)
                                 : launch_split_quant<false>(pr.D, p.cols, tk, tv, p, pr.stream);
}

int run_combine(const Problem &pr, bool after_split) {
    int sms;
    int rc = device_sms(&sms);
    if (rc != FD_OK) return rc;
    fd::CombineParams p;
    p.seqlens = pr.seqlens;
    p.out = pr.out;
    p.lse = pr.lse;
    float *so, *sl;
    int *tickets;
    seg_pointers(pr, &so, &sl, &tickets);
    p.seg_out = so;
    p.seg_lse = sl;
    p.B = pr.B;
    p.Hq = pr.Hq;
    p.Hkv = pr.Hkv;
    p.g = pr.Hq / pr.Hkv;
    p.Lmax = pr.max_len;
    p.P = pr.num_splits;
    return launch_combine(pr.D, p, pr.stream, after_split && pr.max_len > 0);
}

Problem make_problem(int B, int Hq, int Hkv, int D, int max_len, const uint16_t *q, const uint16_t *k,
                     const uint16_t *v, const int32_t *seqlens, float scale, float *out, float *lse, void *ws,
                     size_t ws_bytes, int num_splits, void *stream) {
    Problem pr;
    pr.B = B;
    pr.Hq = Hq;
    pr.Hkv = Hkv;
    pr.D = D;
    pr.max_len = max_len;
    pr.q = q;
    pr.k = k;
    pr.v = v;
    pr.seqlens = seqlens;
    pr.scale = scale;
    pr.out = out;
    pr.lse = lse;
    pr.ws = ws;
    pr.ws_bytes = ws_bytes;
    pr.num_splits = num_splits;
    pr.stream = static_cast<cudaStream_t>(stream);
    return pr;
}

// ------------------------------------------------- fixed scratch buffer --
// Workspace of fd_decode_static: one buffer per device, lives as long as the
// module. Host code must not use the symbol itself as a device address; it
// asks the runtime for the address once per device (static_scratch below).
static __device__ __align__(256) unsigned char g_fd_static_scratch[FD_STATIC_SCRATCH_BYTES];

void *g_static_scratch_ptr[kMaxDevices];
std::mutex g_static_scratch_mutex;

// Device address of this device's fixed scratch buffer, looked up on first
// use. Only a successful lookup is kept: a lookup that fails (for instance
// under stream capture, where loading the module may be refused) returns
// FD_ERR_LAUNCH and is tried again by the next call.
int static_scratch(void **ptr) {
    int dev;
    int rc = current_device(&dev);
    if (rc != FD_OK) return rc;
    std::lock_guard<std::mutex> lock(g_static_scratch_mutex);
    if (g_static_scratch_ptr[dev] == nullptr) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_fd_static_scratch) != cudaSuccess || p == nullptr) {
            cudaGetLastError();
            return FD_ERR_LAUNCH;
        }
        g_static_scratch_ptr[dev] = p;
    }
    *ptr = g_static_scratch_ptr[dev];
    return FD_OK;
}

}  // namespace

extern "C" {

int fd_plan_for_sms(int B, int Hq, int Hkv, int D, int max_len, int num_sms) {
    int rc = check_shape(B, Hq, Hkv, D, max_len);
    if (rc != FD_OK) return rc;
    if (num_sms < 1) return FD_ERR_DEVICE;
    const long long tiles = static_cast<long long>(B) * Hkv * fd::tiles_of(max_len);
    long long want = (tiles + kMinTilesPerSplit - 1) / kMinTilesPerSplit;
    if (want < 1) want = 1;
    if (want > num_sms) want = num_sms;
    // Mid-size batches (at most kMidTilesPerSm tiles per SM): the reduction at
    // the end of the runs weighs more than the last SMs' bandwidth, so use a
    // multiple of 32 splits. Runs then line up with power-of-two row and tile
    // counts, and fewer rows are cut (measured on B200: 8 rows of 128 tiles
    // take 13.7 us with 128 splits, 20.6 us with 148).
    if (num_sms >= 64 && tiles <= static_cast<long long>(kMidTilesPerSm) * num_sms) {
        const long long aligned = num_sms / 32 * 32;
        if (want > aligned) want = aligned;
    }
    if (want > FD_MAX_SPLITS) want = FD_MAX_SPLITS;
    return static_cast<int>(want);
}

int fd_plan(int B, int Hq, int Hkv, int D, int max_len) {
    int rc = check_shape(B, Hq, Hkv, D, max_len);
    if (rc != FD_OK) return rc;
    int sms;
    rc = device_sms(&sms);
    if (rc != FD_OK) return rc;
    return fd_plan_for_sms(B, Hq, Hkv, D, max_len, sms);
}

size_t fd_workspace_bytes(int B, int Hq, int Hkv, int D, int max_len, int num_splits) {
    if (check_shape(B, Hq, Hkv, D, max_len) != FD_OK) return 0;
    if (num_splits < 1 || num_splits > FD_MAX_SPLITS) return 0;
    return workspace_bytes(B, Hq, Hkv, D, num_splits);
}

int fd_decode_splits(int B, int Hq, int Hkv, int D, int max_len, const uint16_t *q, const uint16_t *k_cache,
                     const uint16_t *v_cache, const int32_t *seqlens, float scale, float *out, float *lse,
                     void *workspace, size_t workspace_bytes, int num_splits, void *stream) {
    Problem pr = make_problem(B, Hq, Hkv, D, max_len, q, k_cache, v_cache, seqlens, scale, out, lse, workspace,
                              workspace_bytes, num_splits, stream);
    int rc = check_problem(pr, true);
    if (rc != FD_OK) return rc;
    return run_split(pr, true);
}

int fd_decode(int B, int Hq, int Hkv, int D, int max_len, const uint16_t *q, const uint16_t *k_cache,
              const uint16_t *v_cache, const int32_t *seqlens, float scale, float *out, float *lse,
              void *workspace, size_t workspace_bytes, void *stream) {
    int rc = check_shape(B, Hq, Hkv, D, max_len);
    if (rc != FD_OK) return rc;
    const int S = fd_plan(B, Hq, Hkv, D, max_len);
    if (S < 0) return S;
    return fd_decode_splits(B, Hq, Hkv, D, max_len, q, k_cache, v_cache, seqlens, scale, out, lse, workspace,
                            workspace_bytes, S, stream);
}

int fd_split(int B, int Hq, int Hkv, int D, int max_len, const uint16_t *q, const uint16_t *k_cache,
             const uint16_t *v_cache, const int32_t *seqlens, float scale, float *out, float *lse,
             void *workspace, size_t workspace_bytes, int num_splits, void *stream) {
    Problem pr = make_problem(B, Hq, Hkv, D, max_len, q, k_cache, v_cache, seqlens, scale, out, lse, workspace,
                              workspace_bytes, num_splits, stream);
    int rc = check_problem(pr, true);
    if (rc != FD_OK) return rc;
    return run_split(pr, false);
}

int fd_combine(int B, int Hq, int Hkv, int D, int max_len, const int32_t *seqlens, float *out, float *lse,
               const void *workspace, size_t workspace_bytes, int num_splits, void *stream) {
    Problem pr = make_problem(B, Hq, Hkv, D, max_len, nullptr, nullptr, nullptr, seqlens, 0.f, out, lse,
                              const_cast<void *>(workspace), workspace_bytes, num_splits, stream);
    int rc = check_problem(pr, false);
    if (rc != FD_OK) return rc;
    return run_combine(pr, true);
}

int fd_segments(int B, int Hkv, int max_len, const int32_t *seqlens_host, int num_splits, int32_t *seg_row,
                int32_t *seg_begin, int32_t *seg_end, int32_t *seg_whole, int capacity) {
    if (B < 1 || Hkv < 1 || max_len < 0) return FD_ERR_SHAPE;
    if (static_cast<long long>(B) * Hkv > 0x7fffffffLL) return FD_ERR_SHAPE;
    if (num_splits < 1 || num_splits > FD_MAX_SPLITS) return FD_ERR_SPLITS;
    if (!seqlens_host || !seg_row || !seg_begin || !seg_end || !seg_whole) return FD_ERR_NULL_POINTER;
    const long long slots = num_slots(B, Hkv, num_splits);
    if (slots > 0x7fffffffLL) return FD_ERR_SHAPE;
    if (capacity < slots) return FD_ERR_CAPACITY;
    for (long long s = 0; s < slots; ++s) {
        seg_row[s] = -1;
        seg_begin[s] = seg_end[s] = 0;
        seg_whole[s] = 0;
    }
    long long total = 0;
    for (int b = 0; b < B; ++b) total += fd::tiles_of(fd::clamp_len(seqlens_host[b], max_len));
    const long long N = total * Hkv;
    long long before = 0;
    for (int b = 0; b < B; ++b) {
        const int L = fd::clamp_len(seqlens_host[b], max_len);
        const int n = fd::tiles_of(L);
        for (int h = 0; h < Hkv; ++h) {
            if (n == 0) continue;
            const long long u = static_cast<long long>(b) * Hkv + h;
            const long long first = before * Hkv + static_cast<long long>(h) * n;
            const int i0 = fd::run_of_tile(first, N, num_splits);
            const int i1 = fd::run_of_tile(first + n - 1, N, num_splits);
            for (int i = i0; i <= i1; ++i) {
                const long long lo = fd::run_begin(i, N, num_splits), hi = fd::run_begin(i + 1, N, num_splits);
                if (lo == hi) continue;   // more runs than tiles: this run is empty
                const long long t0 = (lo > first ? lo : first) - first;
                const long long t1 = (hi < first + n ? hi : first + n) - first;
                const long long s = i + u;
                seg_row[s] = static_cast<int32_t>(u);
                seg_begin[s] = static_cast<int32_t>(t0 * fd::kTileTokens);
                const long long e = t1 * fd::kTileTokens;
                seg_end[s] = static_cast<int32_t>(e < L ? e : L);
                seg_whole[s] = i0 == i1 ? 1 : 0;
            }
        }
        before += n;
    }
    return static_cast<int>(slots);
}

int fd_decode_paged(int B, int Hq, int Hkv, int D, int page_size, int num_pages, int max_pages_per_seq,
                    int kv_layout, const uint16_t *q, const uint16_t *k_pages, const uint16_t *v_pages,
                    const int32_t *block_table, const int32_t *seqlens, float scale, float *out, float *lse,
                    void *workspace, size_t workspace_bytes, int num_splits, void *stream) {
    if (page_size < 8 || page_size > 4096 || (page_size & (page_size - 1)) != 0) return FD_ERR_SHAPE;
    if (num_pages < 1 || max_pages_per_seq < 1 || (max_pages_per_seq % 4) != 0) return FD_ERR_SHAPE;
    if (kv_layout != FD_KV_HND && kv_layout != FD_KV_NHD) return FD_ERR_SHAPE;
    const long long max_len = static_cast<long long>(max_pages_per_seq) * page_size;
    if (max_len > 0x7fffffffLL) return FD_ERR_SHAPE;
    int rc = check_shape(B, Hq, Hkv, D, static_cast<int>(max_len));
    if (rc != FD_OK) return rc;
    if (!block_table) return FD_ERR_NULL_POINTER;
    if (!aligned(block_table, 16)) return FD_ERR_ALIGNMENT;
    if (num_splits < 0) return FD_ERR_SPLITS;
    Problem pr = make_problem(B, Hq, Hkv, D, static_cast<int>(max_len), q, k_pages, v_pages, seqlens, scale, out,
                              lse, workspace, workspace_bytes, num_splits == 0 ? 1 : num_splits, stream);
    if ((rc = check_problem(pr, true)) != FD_OK) return rc;   // pointer / alignment checks (no CUDA call)
    if (num_splits == 0) {
        const int S = fd_plan(B, Hq, Hkv, D, static_cast<int>(max_len));
        if (S < 0) return S;
        pr.num_splits = S;
        if ((rc = check_problem(pr, true)) != FD_OK) return rc;   // workspace for the planned count
    }
    // the flattened page coordinate (page * Hkv or page * page_size) must fit in int32
    if (static_cast<long long>(num_pages) * (Hkv > page_size ? Hkv : page_size) > 0x7fffffffLL) return FD_ERR_SHAPE;
    PagedLayout pl{block_table, page_size, num_pages, max_pages_per_seq, kv_layout == FD_KV_NHD};
    return run_split_paged(pr, pl);
}

int fd_decode_quant_paged(int B, int q_len, int Hq, int Hkv, int D, int page_size, int num_pages,
                          int max_pages_per_seq, int kv_layout, int kv_type, const uint16_t *q, const uint8_t *k_pages,
                          const uint8_t *v_pages, const float *k_scale, const float *v_scale,
                          const int32_t *block_table, const int32_t *seqlens, float scale, float *out, float *lse,
                          void *workspace, size_t workspace_bytes, int num_splits, void *stream) {
    if (q_len < 1 || q_len > FD_MAX_GROUP) return FD_ERR_SHAPE;
    if (kv_type != FD_KV_E4M3 && kv_type != FD_KV_INT8) return FD_ERR_SHAPE;
    if (page_size < 8 || page_size > 4096 || (page_size & (page_size - 1)) != 0) return FD_ERR_SHAPE;
    if (num_pages < 1 || max_pages_per_seq < 1 || (max_pages_per_seq % 4) != 0) return FD_ERR_SHAPE;
    if (kv_layout != FD_KV_HND && kv_layout != FD_KV_NHD) return FD_ERR_SHAPE;
    const long long max_len = static_cast<long long>(max_pages_per_seq) * page_size;
    if (max_len > 0x7fffffffLL) return FD_ERR_SHAPE;
    int rc = check_shape(B, Hq, Hkv, D, static_cast<int>(max_len));
    if (rc != FD_OK) return rc;
    if (static_cast<long long>(Hq) * q_len / Hkv > FD_MAX_GROUP) return FD_ERR_GROUP;
    if (!block_table || !k_scale || !v_scale) return FD_ERR_NULL_POINTER;
    if (!aligned(block_table, 16) || !aligned(k_scale, 4) || !aligned(v_scale, 4)) return FD_ERR_ALIGNMENT;
    if (num_splits < 0) return FD_ERR_SPLITS;
    Problem pr = make_problem(B, Hq * q_len, Hkv, D, static_cast<int>(max_len), q,
                              reinterpret_cast<const uint16_t *>(k_pages), reinterpret_cast<const uint16_t *>(v_pages),
                              seqlens, scale, out, lse, workspace, workspace_bytes, num_splits == 0 ? 1 : num_splits,
                              stream);
    if ((rc = check_problem(pr, true)) != FD_OK) return rc;
    if (num_splits == 0) {
        const int S = fd_plan(B, Hq, Hkv, D, static_cast<int>(max_len));
        if (S < 0) return S;
        pr.num_splits = S;
        if ((rc = check_problem(pr, true)) != FD_OK) return rc;
    }
    pr.Hq = Hq;
    if (static_cast<long long>(num_pages) * (Hkv > page_size ? Hkv : page_size) > 0x7fffffffLL) return FD_ERR_SHAPE;
    PagedLayout pl{block_table, page_size, num_pages, max_pages_per_seq, kv_layout == FD_KV_NHD};
    return run_split_paged(pr, pl, q_len, kv_type, k_scale, v_scale);
}

int fd_decode_multi(int B, int q_len, int Hq, int Hkv, int D, int max_len, const uint16_t *q,
                    const uint16_t *k_cache, const uint16_t *v_cache, const int32_t *seqlens, float scale, float *out,
                    float *lse, void *workspace, size_t workspace_bytes, int num_splits, void *stream) {
    if (q_len < 1 || q_len > FD_MAX_GROUP) return FD_ERR_SHAPE;
    int rc = check_shape(B, Hq, Hkv, D, max_len);
    if (rc != FD_OK) return rc;
    if (static_cast<long long>(Hq) * q_len / Hkv > FD_MAX_GROUP) return FD_ERR_GROUP;
    if (num_splits < 0) return FD_ERR_SPLITS;
    // the workspace and the checks see the (query, head) columns as Hq * q_len query heads
    const int Hqq = Hq * q_len;
    Problem pr = make_problem(B, Hqq, Hkv, D, max_len, q, k_cache, v_cache, seqlens, scale, out, lse, workspace,
                              workspace_bytes, num_splits == 0 ? 1 : num_splits, stream);
    if ((rc = check_problem(pr, true)) != FD_OK) return rc;
    if (num_splits == 0) {
        const int S = fd_plan(B, Hq, Hkv, D, max_len);
        if (S < 0) return S;
        pr.num_splits = S;
        if ((rc = check_problem(pr, true)) != FD_OK) return rc;
    }
    pr.Hq = Hq;   // the kernel indexes q / out with the real head count
    return run_split(pr, true, q_len);
}

int fd_decode_quant(int B, int q_len, int Hq, int Hkv, int D, int max_len, int kv_type, const uint16_t *q,
                    const uint8_t *k_codes, const uint8_t *v_codes, const float *k_scale, const float *v_scale,
                    const int32_t *seqlens, float scale, float *out, float *lse, void *workspace,
                    size_t workspace_bytes, int num_splits, void *stream) {
    if (q_len < 1 || q_len > FD_MAX_GROUP) return FD_ERR_SHAPE;
    if (kv_type != FD_KV_E4M3 && kv_type != FD_KV_INT8) return FD_ERR_SHAPE;
    int rc = check_shape(B, Hq, Hkv, D, max_len);
    if (rc != FD_OK) return rc;
    if (static_cast<long long>(Hq) * q_len / Hkv > FD_MAX_GROUP) return FD_ERR_GROUP;
    if (num_splits < 0) return FD_ERR_SPLITS;
    if (max_len > 0) {
        if (!k_scale || !v_scale) return FD_ERR_NULL_POINTER;
        if (!aligned(k_scale, 4) || !aligned(v_scale, 4)) return FD_ERR_ALIGNMENT;
    }
    // the checks and the workspace see the (query, head) columns as Hq * q_len heads
    const int Hqq = Hq * q_len;
    Problem pr = make_problem(B, Hqq, Hkv, D, max_len, q, reinterpret_cast<const uint16_t *>(k_codes),
                              reinterpret_cast<const uint16_t *>(v_codes), seqlens, scale, out, lse, workspace,
                              workspace_bytes, num_splits == 0 ? 1 : num_splits, stream);
    if ((rc = check_problem(pr, true)) != FD_OK) return rc;
    if (num_splits == 0) {
        const int S = fd_plan(B, Hq, Hkv, D, max_len);
        if (S < 0) return S;
        pr.num_splits = S;
        if ((rc = check_problem(pr, true)) != FD_OK) return rc;
    }
    pr.Hq = Hq;
    return run_split_quant(pr, q_len, kv_type, k_scale, v_scale);
}

int fd_merge_partials(int R, int rows, int D, const float *part_out, const float *part_lse, float *out, float *lse,
                      void *stream) {
    if (R < 1 || rows < 0) return FD_ERR_SHAPE;
    if (D < 4 || D > 4096 || D % 4 != 0) return FD_ERR_HEAD_DIM;
    if (rows == 0) return FD_OK;
    if (!part_out || !part_lse || !out || !lse) return FD_ERR_NULL_POINTER;
    if (!aligned(part_out, 16) || !aligned(out, 16) || !aligned(part_lse, 4) || !aligned(lse, 4))
        return FD_ERR_ALIGNMENT;
    int dev;
    if (current_device(&dev) != FD_OK) return FD_ERR_DEVICE;
    const long long items = static_cast<long long>(rows) * (D / 4);
    const long long blocks = (items + fd::kPartialsThreads - 1) / fd::kPartialsThreads;
    if (inject_launch_failure()) return FD_ERR_LAUNCH;
    fd::fd_merge_partials_kernel<<<static_cast<unsigned>(blocks), fd::kPartialsThreads, 0,
                                   static_cast<cudaStream_t>(stream)>>>(part_out, part_lse, R, rows, D, out, lse);
    if (cudaGetLastError() != cudaSuccess) return FD_ERR_LAUNCH;
    return FD_OK;
}

int fd_decode_static(int B, int Hq, int Hkv, int D, int max_len, const uint16_t *q, const uint16_t *k_cache,
                     const uint16_t *v_cache, const int32_t *seqlens, float scale, float *out, float *lse,
                     void *stream) {
    // argument checks first (no CUDA call): validate as an unsplit call, which needs no workspace
    Problem pr = make_problem(B, Hq, Hkv, D, max_len, q, k_cache, v_cache, seqlens, scale, out, lse, nullptr, 0, 1,
                              stream);
    int rc = check_problem(pr, true);
    if (rc != FD_OK) return rc;
    const int S = fd_plan(B, Hq, Hkv, D, max_len);
    if (S < 0) return S;
    const WorkspaceLayout w = workspace_layout(B, Hq, Hkv, D, S);
    if (w.total > FD_STATIC_SCRATCH_BYTES) return FD_ERR_STATIC_LIMIT;
    void *scratch = nullptr;
    if (w.total > 0) {
        if ((rc = static_scratch(&scratch)) != FD_OK) return rc;
        // the per-row counters must start at zero; the segments need no clearing
        char *tickets = static_cast<char *>(scratch) + w.tickets;
        if (cudaMemsetAsync(tickets, 0, w.total - w.tickets, static_cast<cudaStream_t>(stream)) != cudaSuccess) {
            cudaGetLastError();
            return FD_ERR_LAUNCH;
        }
    }
    pr.ws = scratch;
    pr.ws_bytes = w.total;
    pr.num_splits = S;
    return run_split(pr, true);
}

int fd_workspace_init(void *workspace, size_t workspace_bytes, void *stream) {
    if (workspace_bytes == 0) return FD_OK;
    if (!workspace) return FD_ERR_NULL_POINTER;
    int dev;
    if (current_device(&dev) != FD_OK) return FD_ERR_DEVICE;
    if (cudaMemsetAsync(workspace, 0, workspace_bytes, static_cast<cudaStream_t>(stream)) != cudaSuccess) {
        cudaGetLastError();
        return FD_ERR_LAUNCH;
    }
    return FD_OK;
}

int fd_device_status(void *stream) {
    int dev;
    if (current_device(&dev) != FD_OK) return FD_ERR_DEVICE;
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) {
        cudaGetLastError();
        return FD_ERR_LAUNCH;
    }
    int word = 0;
    const int zero = 0;
    if (cudaMemcpyFromSymbol(&word, fd::g_fd_error_word, sizeof word) != cudaSuccess ||
        cudaMemcpyToSymbol(fd::g_fd_error_word, &zero, sizeof zero) != cudaSuccess) {
        cudaGetLastError();
        return FD_ERR_LAUNCH;
    }
    return word;
}

const char *fd_strerror(int code) {
    switch (code) {
        case FD_OK: return "ok";
        case FD_ERR_NULL_POINTER: return "a required pointer is NULL";
        case FD_ERR_SHAPE: return "invalid or too large B / Hq / Hkv / max_len";
        case FD_ERR_GROUP: return "Hq must be a multiple of Hkv with Hq/Hkv <= 16";
        case FD_ERR_HEAD_DIM: return "head dimension D must be 64 or 128";
        case FD_ERR_ALIGNMENT: return "pointer misaligned (q/k/v/out/workspace need 16 bytes, seqlens/lse 4)";
        case FD_ERR_WORKSPACE: return "workspace missing or smaller than fd_workspace_bytes()";
        case FD_ERR_SPLITS: return "num_splits out of range [1, 65535]";
        case FD_ERR_DEVICE: return "no usable CUDA device of compute capability 10.0";
        case FD_ERR_LAUNCH: return "kernel launch or tensor-map encoding failed";
        case FD_ERR_TIMEOUT: return "a device-side wait gave up; outputs of that call are invalid";
        case FD_ERR_CAPACITY: return "output arrays too small";
        case FD_ERR_STATIC_LIMIT:
            return "problem needs more scratch than fd_decode_static's fixed 8 MiB buffer; use fd_decode with a workspace";
        case FD_ERR_BOUNDS: return "a debug build's device-side bounds check failed; outputs of that call are invalid";
        default: return "unknown error code";
    }
}

int fd_version(void) { return kVersion; }

}  // extern "C"
