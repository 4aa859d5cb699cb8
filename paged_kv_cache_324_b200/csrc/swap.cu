// pkv_swap_blocks: block-granular copy between two pools of the same layout,
// one of which is typically pinned host memory (the "vLLM and PagedAttention"
// transcript, on preemption: a group's KV data moves to CPU memory and is
// brought back later; the transfer rate is the cost).
//
// One launch moves every listed block of the K and V pools.  Host memory is
// reached through its device mapping (zero copy), so the kernel itself drives
// the link: each thread keeps four 16-byte loads in flight before its stores,
// and the grid covers the SMs several times over, so that enough requests are
// outstanding to hide the link's latency.

#include <cuda_runtime.h>

#include "pkv_device.cuh"
#include "pkv_host.h"

namespace pkv {
namespace {

constexpr int kSwapThreads = 256;
constexpr int kSwapUnroll = 4;

// Flat index over (pool, pair, 16-byte vector): consecutive threads take consecutive
// vectors of one block, so every warp reads and writes 512 contiguous bytes.
__global__ void __launch_bounds__(kSwapThreads)
swap_blocks_kernel(const uint8_t* src_k, const uint8_t* src_v, uint8_t* dst_k, uint8_t* dst_v, size_t block_bytes,
                   const int64_t* pairs, int num_pairs, int src_blocks, int dst_blocks, uint32_t* err) {
    // plain (coherent) loads throughout: any operand may live in mapped host memory
    pdl_trigger();
    pdl_wait();   // the previous kernel may still use either pool
    const size_t nvec = block_bytes / 16;
    const size_t per_pool = nvec * static_cast<size_t>(num_pairs);
    const size_t total = 2 * per_pool;
    const size_t stride = static_cast<size_t>(gridDim.x) * blockDim.x;
    for (size_t base = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; base < total;
         base += stride * kSwapUnroll) {
        uint4 v[kSwapUnroll];
        uint4* d[kSwapUnroll];
#pragma unroll
        for (int u = 0; u < kSwapUnroll; ++u) {
            d[u] = nullptr;
            const size_t i = base + u * stride;
            if (i >= total) continue;
            const bool is_v = i >= per_pool;
            const size_t r = is_v ? i - per_pool : i;
            const size_t p = r / nvec, e = r - p * nvec;
            const long long s = pairs[2 * p], t = pairs[2 * p + 1];
            if (s < 0 || s >= src_blocks || t < 0 || t >= dst_blocks) {
                if (e == 0 && !is_v) raise_error(err, PKV_DEVERR_PAIR);
                continue;
            }
            const uint8_t* sp = (is_v ? src_v : src_k) + static_cast<size_t>(s) * block_bytes;
            uint8_t* dp = (is_v ? dst_v : dst_k) + static_cast<size_t>(t) * block_bytes;
            v[u] = reinterpret_cast<const uint4*>(sp)[e];
            d[u] = reinterpret_cast<uint4*>(dp) + e;
        }
#pragma unroll
        for (int u = 0; u < kSwapUnroll; ++u)
            if (d[u]) *d[u] = v[u];
    }
}

// A pool the kernel may touch: device memory, or host memory that CUDA pinned and mapped
// into the device's address space under the same address (pageable memory would fault).
bool device_reachable(const void* p) {
    cudaPointerAttributes at{};
    if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    if (at.type == cudaMemoryTypeDevice || at.type == cudaMemoryTypeManaged) return true;
    return at.type == cudaMemoryTypeHost && at.devicePointer == p;
}

}  // namespace
}  // namespace pkv

extern "C" pkv_status pkv_swap_blocks(const void* src_k_pool, const void* src_v_pool, int src_num_blocks,
                                      void* dst_k_pool, void* dst_v_pool, int dst_num_blocks, size_t block_bytes,
                                      const int64_t* pairs, int num_pairs, uint32_t* device_error, void* stream) {
    using namespace pkv;
    if (num_pairs < 0 || src_num_blocks <= 0 || dst_num_blocks <= 0 || block_bytes == 0) return PKV_ERR_INVALID_ARG;
    if (block_bytes % 16 != 0) return PKV_ERR_UNSUPPORTED;
    if (num_pairs == 0) return PKV_OK;
    if (!src_k_pool || !src_v_pool || !dst_k_pool || !dst_v_pool || !pairs) return PKV_ERR_INVALID_ARG;
    if (!aligned16(src_k_pool) || !aligned16(src_v_pool) || !aligned16(dst_k_pool) || !aligned16(dst_v_pool) ||
        (reinterpret_cast<uintptr_t>(pairs) & 7))
        return PKV_ERR_ALIGNMENT;
    if (!device_reachable(src_k_pool) || !device_reachable(src_v_pool) || !device_reachable(dst_k_pool) ||
        !device_reachable(dst_v_pool) || !device_reachable(pairs))
        return PKV_ERR_INVALID_ARG;
    const size_t total = 2 * (block_bytes / 16) * static_cast<size_t>(num_pairs);
    size_t blocks = (total + kSwapThreads * kSwapUnroll - 1) / (kSwapThreads * kSwapUnroll);
    const size_t cap = static_cast<size_t>(num_sms()) * 8;
    if (blocks > cap) blocks = cap;
    const cudaError_t e = launch_pdl(swap_blocks_kernel, dim3(static_cast<unsigned>(blocks)), dim3(kSwapThreads), 0,
                                     static_cast<cudaStream_t>(stream), static_cast<const uint8_t*>(src_k_pool),
                                     static_cast<const uint8_t*>(src_v_pool), static_cast<uint8_t*>(dst_k_pool),
                                     static_cast<uint8_t*>(dst_v_pool), block_bytes, pairs, num_pairs, src_num_blocks,
                                     dst_num_blocks, device_error);
    return e == cudaSuccess ? PKV_OK : PKV_ERR_CUDA;
}
