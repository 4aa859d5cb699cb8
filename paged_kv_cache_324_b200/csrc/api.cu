// Library-wide entry points: version, status strings, and the host helpers
// the launchers share.
#include <cuda_runtime.h>

#include <algorithm>
#include <mutex>
#include <vector>

#include "pkv_device.cuh"
#include "pkv_host.h"

namespace pkv {

int num_sms() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 148;
    return n;
}

long long l2_bytes() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 126ll << 20;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrL2CacheSize, dev) != cudaSuccess || n <= 0) return 126ll << 20;
    return n;
}

EncodeTiledFn encode_tiled_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q{};
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

}  // namespace pkv

extern "C" int pkv_version(void) { return 100; }

extern "C" const char* pkv_status_string(pkv_status s) {
    switch (s) {
    case PKV_OK: return "ok";
    case PKV_ERR_INVALID_ARG: return "invalid argument";
    case PKV_ERR_UNSUPPORTED: return "unsupported size or dtype combination";
    case PKV_ERR_WORKSPACE: return "workspace missing or too small";
    case PKV_ERR_CUDA: return "CUDA error";
    case PKV_ERR_ALIGNMENT: return "pointer not 16-byte aligned";
    case PKV_ERR_OUT_OF_BLOCKS: return "out of free blocks";
    }
    return "unknown status";
}

// ---- host check of a block-pair list (copy-on-write, swap) ----------------------------

extern "C" pkv_status pkv_check_block_pairs(const int64_t* pairs, int num_pairs, int src_num_blocks,
                                            int dst_num_blocks, int same_pool) {
    if (num_pairs < 0 || src_num_blocks <= 0 || dst_num_blocks <= 0) return PKV_ERR_INVALID_ARG;
    if (num_pairs == 0) return PKV_OK;
    if (!pairs) return PKV_ERR_INVALID_ARG;
    std::vector<int64_t> dst(static_cast<size_t>(num_pairs));
    for (int i = 0; i < num_pairs; ++i) {
        const int64_t s = pairs[2 * static_cast<size_t>(i)], d = pairs[2 * static_cast<size_t>(i) + 1];
        if (s < 0 || s >= src_num_blocks || d < 0 || d >= dst_num_blocks) return PKV_ERR_INVALID_ARG;
        dst[static_cast<size_t>(i)] = d;
    }
    std::sort(dst.begin(), dst.end());
    if (std::adjacent_find(dst.begin(), dst.end()) != dst.end()) return PKV_ERR_INVALID_ARG;
    if (same_pool) {
        for (int i = 0; i < num_pairs; ++i)
            if (std::binary_search(dst.begin(), dst.end(), pairs[2 * static_cast<size_t>(i)]))
                return PKV_ERR_INVALID_ARG;
    }
    return PKV_OK;
}

// ---- diagnostic: one bounded wait that nothing completes ---------------------------

namespace pkv {
namespace {

// Waits on phase 0 of a fresh barrier that no thread arrives on; the wait gives up
// after timeout_ns and reports PKV_DEVERR_TIMEOUT, exercising the same bounded
// wait the decode kernel uses for its TMA and ring barriers.
__global__ void selftest_wait_kernel(uint32_t* err, unsigned long long timeout_ns) {
    __shared__ __align__(8) uint64_t bar;
    const uint32_t b = smem_addr(&bar);
    if (threadIdx.x == 0) {
        mbar_init(b, 1);
        mbar_fence_init();
    }
    __syncthreads();
    if (threadIdx.x == 0 && !mbar_wait(b, 0, global_timer_ns() + timeout_ns)) raise_error(err, PKV_DEVERR_TIMEOUT);
}

}  // namespace
}  // namespace pkv

extern "C" pkv_status pkv_selftest_bounded_wait(uint32_t* device_error, unsigned timeout_us, void* stream) {
    if (!device_error || timeout_us == 0 || timeout_us > 10u * 1000u * 1000u) return PKV_ERR_INVALID_ARG;
    pkv::selftest_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
        device_error, static_cast<unsigned long long>(timeout_us) * 1000ull);
    return cudaGetLastError() == cudaSuccess ? PKV_OK : PKV_ERR_CUDA;
}
