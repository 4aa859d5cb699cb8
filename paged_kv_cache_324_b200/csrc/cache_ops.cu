// pkv_reshape_and_cache and pkv_copy_blocks: the two memory kernels of a
// decode step.
//
// reshape_and_cache writes each new token's K/V rows into the pool slot the
// block table gives it (Ultralytics glossary "PagedAttention", section "How
// paging works": pool[table[pos / B], pos % B] = key).  copy_blocks is the
// block-granular copy-on-write of shared blocks (glossary, section "Sharing
// blocks across sequences"; the "vLLM and PagedAttention" transcript says the
// partially filled shared block is the one that gets copied).
//
// Both are HBM-bound byte movers: one thread moves one 16-byte vector (8
// elements in, 8 elements out), consecutive threads cover consecutive
// vectors of a token's row so loads and stores coalesce, and the grid is a
// multiple of the SM count with a grid-stride loop.

#include <cmath>

#include <cuda_runtime.h>

#include "pkv_device.cuh"
#include "pkv_host.h"

namespace pkv {
namespace {

// ---- reshape_and_cache -------------------------------------------------------

template <bool kFp8, bool kBf16In>
__global__ void __launch_bounds__(256)
reshape_and_cache_kernel(const uint4* __restrict__ k, const uint4* __restrict__ v,
                         uint8_t* __restrict__ k_pool, uint8_t* __restrict__ v_pool,
                         const int64_t* __restrict__ slot_mapping, int num_tokens,
                         int num_kv_heads, int head_dim, int block_size, int num_blocks,
                         float k_scale, float v_scale, uint32_t* err) {
    pdl_trigger();
    pdl_wait();   // the previous kernel may still read the pool
    const int vec_per_row = head_dim / 8;                 // 8 elements per 16-byte input vector
    const int vec_per_tok = num_kv_heads * vec_per_row;
    const long long total = static_cast<long long>(num_tokens) * vec_per_tok;
    const long long limit = static_cast<long long>(num_blocks) * block_size;
    constexpr int kOutElem = kFp8 ? 1 : 2;
    for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < total;
         i += static_cast<long long>(gridDim.x) * blockDim.x) {
        const int t = static_cast<int>(i / vec_per_tok);
        const int rem = static_cast<int>(i - static_cast<long long>(t) * vec_per_tok);
        const int h = rem / vec_per_row;
        const int vec = rem - h * vec_per_row;
        const long long slot = __ldg(slot_mapping + t);
        if (slot < 0) continue;
        if (slot >= limit) {
            if (rem == 0) raise_error(err, PKV_DEVERR_SLOT);
            continue;
        }
        const long long blk = slot / block_size;
        const int off = static_cast<int>(slot - blk * block_size);
        const size_t dst_elem =
            ((static_cast<size_t>(blk) * num_kv_heads + h) * block_size + off) * head_dim + vec * 8;
        const uint4 kx = __ldg(k + i);
        const uint4 vx = __ldg(v + i);
        if constexpr (!kFp8) {
            *reinterpret_cast<uint4*>(k_pool + dst_elem * kOutElem) = kx;
            *reinterpret_cast<uint4*>(v_pool + dst_elem * kOutElem) = vx;
        } else {
            // x / scale in IEEE float32, then E4M3 round-to-nearest-even saturating at +-448.
            auto quant8 = [](uint4 x, float s) {
                const uint32_t w[4] = {x.x, x.y, x.z, x.w};
                uint32_t packed[2] = {0u, 0u};
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    float lo, hi;
                    if constexpr (kBf16In) {
                        lo = __uint_as_float(w[j] << 16);
                        hi = __uint_as_float(w[j] & 0xffff0000u);
                    } else {
                        __half2 hh = *reinterpret_cast<const __half2*>(&w[j]);
                        float2 f = __half22float2(hh);
                        lo = f.x;
                        hi = f.y;
                    }
                    float2 q = make_float2(__fdiv_rn(lo, s), __fdiv_rn(hi, s));
                    __nv_fp8x2_storage_t b = __nv_cvt_float2_to_fp8x2(q, __NV_SATFINITE, __NV_E4M3);
                    packed[j >> 1] |= static_cast<uint32_t>(b) << ((j & 1) * 16);
                }
                return make_uint2(packed[0], packed[1]);
            };
            *reinterpret_cast<uint2*>(k_pool + dst_elem) = quant8(kx, k_scale);
            *reinterpret_cast<uint2*>(v_pool + dst_elem) = quant8(vx, v_scale);
        }
    }
}

// ---- copy_blocks ---------------------------------------------------------------

// grid.x strides over 16-byte vectors of a block, grid.y over pairs, grid.z = K / V pool.
__global__ void __launch_bounds__(256)
copy_blocks_kernel(uint8_t* __restrict__ k_pool, uint8_t* __restrict__ v_pool,
                   size_t block_bytes, const int64_t* __restrict__ pairs, int num_pairs,
                   int num_blocks, uint32_t* err) {
    pdl_trigger();
    pdl_wait();   // the previous kernel may still read the pool
    uint8_t* pool = blockIdx.z == 0 ? k_pool : v_pool;
    const size_t nvec = block_bytes / 16;
    for (int p = blockIdx.y; p < num_pairs; p += gridDim.y) {
        const long long src = __ldg(pairs + 2 * p);
        const long long dst = __ldg(pairs + 2 * p + 1);
        if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks) {
            if (blockIdx.x == 0 && blockIdx.z == 0 && threadIdx.x == 0) raise_error(err, PKV_DEVERR_PAIR);
            continue;
        }
        const uint4* s = reinterpret_cast<const uint4*>(pool + static_cast<size_t>(src) * block_bytes);
        uint4* d = reinterpret_cast<uint4*>(pool + static_cast<size_t>(dst) * block_bytes);
        for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < nvec;
             i += static_cast<size_t>(gridDim.x) * blockDim.x)
            d[i] = s[i];
    }
}

}  // namespace
}  // namespace pkv

extern "C" pkv_status pkv_reshape_and_cache(const void* k, const void* v, pkv_dtype in_dtype,
                                            void* k_pool, void* v_pool, pkv_dtype kv_dtype,
                                            float k_scale, float v_scale,
                                            const int64_t* slot_mapping, int num_tokens,
                                            int num_kv_heads, int head_dim, int block_size,
                                            int num_blocks, uint32_t* device_error, void* stream) {
    using namespace pkv;
    if (num_tokens < 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 || num_blocks <= 0)
        return PKV_ERR_INVALID_ARG;
    if (in_dtype != PKV_F16 && in_dtype != PKV_BF16) return PKV_ERR_UNSUPPORTED;
    if (kv_dtype != in_dtype && kv_dtype != PKV_FP8_E4M3) return PKV_ERR_UNSUPPORTED;
    if (head_dim % 8 != 0) return PKV_ERR_UNSUPPORTED;
    if (num_tokens == 0) return PKV_OK;
    if (!k || !v || !k_pool || !v_pool || !slot_mapping) return PKV_ERR_INVALID_ARG;
    if (kv_dtype == PKV_FP8_E4M3 &&
        !(k_scale > 0.f && v_scale > 0.f && std::isfinite(k_scale) && std::isfinite(v_scale)))
        return PKV_ERR_INVALID_ARG;
    if (!aligned16(k) || !aligned16(v) || !aligned16(k_pool) || !aligned16(v_pool) ||
        (reinterpret_cast<uintptr_t>(slot_mapping) & 7))
        return PKV_ERR_ALIGNMENT;
    const long long vecs = static_cast<long long>(num_tokens) * num_kv_heads * (head_dim / 8);
    const int threads = 256;
    long long blocks = (vecs + threads - 1) / threads;
    const long long cap = static_cast<long long>(num_sms()) * 8;
    if (blocks > cap) blocks = cap;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const bool fp8 = kv_dtype == PKV_FP8_E4M3, bf16 = in_dtype == PKV_BF16;
    auto launch = [&](auto kern) {
        return launch_pdl(kern, dim3(static_cast<unsigned>(blocks)), dim3(threads), 0, st,
                          static_cast<const uint4*>(k), static_cast<const uint4*>(v), static_cast<uint8_t*>(k_pool),
                          static_cast<uint8_t*>(v_pool), slot_mapping, num_tokens, num_kv_heads, head_dim,
                          block_size, num_blocks, k_scale, v_scale, device_error);
    };
    cudaError_t e;
    if (!fp8)
        e = launch(reshape_and_cache_kernel<false, false>);
    else if (bf16)
        e = launch(reshape_and_cache_kernel<true, true>);
    else
        e = launch(reshape_and_cache_kernel<true, false>);
    return e == cudaSuccess ? PKV_OK : PKV_ERR_CUDA;
}

extern "C" pkv_status pkv_copy_blocks(void* k_pool, void* v_pool, size_t block_bytes,
                                      const int64_t* pairs, int num_pairs, int num_blocks,
                                      uint32_t* device_error, void* stream) {
    using namespace pkv;
    if (num_pairs < 0 || num_blocks <= 0 || block_bytes == 0) return PKV_ERR_INVALID_ARG;
    if (block_bytes % 16 != 0) return PKV_ERR_UNSUPPORTED;
    if (num_pairs == 0) return PKV_OK;
    if (!k_pool || !v_pool || !pairs) return PKV_ERR_INVALID_ARG;
    if (!aligned16(k_pool) || !aligned16(v_pool) || (reinterpret_cast<uintptr_t>(pairs) & 7))
        return PKV_ERR_ALIGNMENT;
    const size_t nvec = block_bytes / 16;
    const int threads = 256;
    unsigned gx = static_cast<unsigned>((nvec + threads * 2 - 1) / (threads * 2));  // 2 vectors per thread
    if (gx == 0) gx = 1;
    unsigned gy = static_cast<unsigned>(num_pairs < 65535 ? num_pairs : 65535);
    dim3 grid(gx, gy, 2);
    const cudaError_t e = launch_pdl(copy_blocks_kernel, grid, dim3(threads), 0, static_cast<cudaStream_t>(stream),
                                     static_cast<uint8_t*>(k_pool), static_cast<uint8_t*>(v_pool), block_bytes,
                                     pairs, num_pairs, num_blocks, device_error);
    return e == cudaSuccess ? PKV_OK : PKV_ERR_CUDA;
}
