// pkv_stream_read: a read-only pass over a device buffer, the denominator that
// a read-mostly kernel such as paged decode attention is measured against.
//
// Decode attention reads the KV cache and writes almost nothing, so a copy
// (half reads, half writes) understates what HBM delivers to it.  This kernel
// reads every 16-byte vector of the buffer once, with non-allocating loads that
// bypass L1 and an evict-first L2 hint, folds them into one 32-bit value per
// thread and keeps them alive by a data-dependent store that (for any real
// buffer) never happens.  Each thread keeps four loads in flight; the grid is a
// fixed number of CTAs per SM with a grid-stride loop, so every SM streams
// until the end.

#include <cuda_runtime.h>

#include "pkv_device.cuh"
#include "pkv_host.h"

namespace pkv {
namespace {

constexpr int kReadThreads = 512;
constexpr int kReadCtasPerSm = 4;
constexpr int kReadUnroll = 4;

__device__ __forceinline__ uint4 ld_stream(const uint4* p, uint64_t policy) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.L2::cache_hint.v4.u32 {%0, %1, %2, %3}, [%4], %5;"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p), "l"(policy));
    return v;
}

__global__ void __launch_bounds__(kReadThreads) stream_read_kernel(const uint4* __restrict__ p, size_t n,
                                                                   uint32_t* sink) {
    const uint64_t pol = l2_policy_evict_first();
    const size_t stride = static_cast<size_t>(gridDim.x) * blockDim.x;
    size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x;
    uint32_t acc = 0;
    for (; i + (kReadUnroll - 1) * stride < n; i += kReadUnroll * stride) {
        uint4 v[kReadUnroll];
#pragma unroll
        for (int u = 0; u < kReadUnroll; ++u) v[u] = ld_stream(p + i + u * stride, pol);
#pragma unroll
        for (int u = 0; u < kReadUnroll; ++u) acc += v[u].x ^ v[u].y ^ v[u].z ^ v[u].w;
    }
    for (; i < n; i += stride) {
        const uint4 v = ld_stream(p + i, pol);
        acc += v.x ^ v.y ^ v.z ^ v.w;
    }
    if (acc == 0x9e3779b9u && sink) atomicAdd(sink, 1u);   // keeps the loads; practically never taken
}

}  // namespace
}  // namespace pkv

extern "C" pkv_status pkv_stream_read(const void* buf, size_t bytes, uint32_t* sink, void* stream) {
    using namespace pkv;
    if (bytes == 0) return PKV_OK;
    if (!buf) return PKV_ERR_INVALID_ARG;
    if (!aligned16(buf) || bytes % 16 != 0 || (reinterpret_cast<uintptr_t>(sink) & 3)) return PKV_ERR_ALIGNMENT;
    const dim3 grid(static_cast<unsigned>(num_sms() * kReadCtasPerSm));
    stream_read_kernel<<<grid, kReadThreads, 0, static_cast<cudaStream_t>(stream)>>>(
        static_cast<const uint4*>(buf), bytes / 16, sink);
    return cudaGetLastError() == cudaSuccess ? PKV_OK : PKV_ERR_CUDA;
}
