// pkv_paged_attn_prefill_fp8: chunked prefill over an E4M3 cache (Ultralytics glossary
// "PagedAttention", section "Related methods": an 8-bit KV cache).
//
// Prefill is bound by the tensor cores, not by the cache bytes (each K/V tile is used by
// 2 x 128 query rows), so the FP8 case reuses the 16-bit tensor-core kernel: a gather kernel
// first widens the blocks each sequence's queries can reach into 16-bit workspace pools laid
// out one row of max_blocks_per_seq blocks per sequence, with a block table of their own.  E4M3
// values are exactly representable in f16 and bf16, so both are widened exactly: K to the
// query's type, its scale folded into the softmax scale; V to f16, its scale applied to the
// output rows, so that P.V is one f16 product for either query type.  A block id outside the
// pool becomes an out-of-range entry of the workspace table, which the prefill kernel reports
// (PKV_DEVERR_BLOCK_ID) with NaN rows, as for a 16-bit cache.

#include <cmath>
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "pkv_device.cuh"
#include "pkv_host.h"

namespace pkv {
namespace {

constexpr int kWidenThreads = 256;
constexpr int kWidenUnroll = 4;

// Two E4M3 values (low byte first) -> two f16 values in one word (exact).
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint16_t x) {
    uint32_t h;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h) : "h"(x));
    return h;
}

// Two f16 values -> the same two values as bf16 (exact for widened E4M3: 4 significant bits).
__device__ __forceinline__ uint32_t f16x2_to_bf16x2(uint32_t f16x2) {
    const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&f16x2));
    const __nv_bfloat162 b = __floats2bfloat162_rn(f.x, f.y);
    return *reinterpret_cast<const uint32_t*>(&b);
}

// 8 E4M3 bytes -> 8 f16 (or bf16) values, one 16-byte vector (exact).
template <bool kBf16>
__device__ __forceinline__ uint4 widen8(const uint2& x) {
    const uint32_t w[2] = {x.x, x.y};
    uint32_t o[4];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const uint32_t a = e4m3x2_to_f16x2(static_cast<uint16_t>(w[i] & 0xffffu));
        const uint32_t b = e4m3x2_to_f16x2(static_cast<uint16_t>(w[i] >> 16));
        o[2 * i] = kBf16 ? f16x2_to_bf16x2(a) : a;
        o[2 * i + 1] = kBf16 ? f16x2_to_bf16x2(b) : b;
    }
    return make_uint4(o[0], o[1], o[2], o[3]);
}

// Flat index over (sequence s, table slot j, 8-byte unit of the E4M3 block): block s * maxb + j
// of the workspace pools receives the widened block block_tables[s][j], for j < ceil(L_s / B):
// K in the query's type (kBf16), V in f16.
// Each thread reads 8 bytes and writes the 16-byte vector they widen to, so a warp's loads and
// stores each cover one contiguous run (256 and 512 bytes).
template <bool kBf16>
__global__ void __launch_bounds__(kWidenThreads)
widen_blocks_kernel(const uint2* __restrict__ k_pool, const uint2* __restrict__ v_pool, uint4* __restrict__ wk,
                    uint4* __restrict__ wv, int32_t* __restrict__ wtab, const int32_t* __restrict__ tables,
                    const int32_t* __restrict__ lens, int num_seqs, int maxb, long long units_per_block,
                    int block_size, int num_blocks, uint32_t* err) {
    pdl_trigger();
    pdl_wait();   // the pool may still be written by the previous kernel (the chunk's scatter)
    const long long total = static_cast<long long>(num_seqs) * maxb * units_per_block;
    const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
    const long long cap = static_cast<long long>(maxb) * block_size;
    // kWidenUnroll units per thread and round: their table entries, then their K and V loads, are all in
    // flight before the first conversion
    for (long long base = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; base < total;
         base += stride * kWidenUnroll) {
        long long src[kWidenUnroll];
#pragma unroll
        for (int u = 0; u < kWidenUnroll; ++u) {
            src[u] = -1;
            const long long i = base + u * stride;
            if (i >= total) continue;
            const long long blk = i / units_per_block;
            const long long e = i - blk * units_per_block;
            const int s = static_cast<int>(blk / maxb), j = static_cast<int>(blk - static_cast<long long>(s) * maxb);
            const int L = __ldg(lens + s);
            const int nb = L <= 0 ? 0 : static_cast<int>((min(static_cast<long long>(L), cap) + block_size - 1) / block_size);
            if (j >= nb) continue;
            const int pid = __ldg(tables + blk);
            const bool bad = pid < 0 || pid >= num_blocks;
            if (e == 0) {
                wtab[blk] = bad ? -1 : static_cast<int32_t>(blk);
                if (bad) raise_error(err, PKV_DEVERR_BLOCK_ID);
            }
            if (!bad) src[u] = static_cast<long long>(pid) * units_per_block + e;
        }
        uint2 kx[kWidenUnroll], vx[kWidenUnroll];
#pragma unroll
        for (int u = 0; u < kWidenUnroll; ++u)
            if (src[u] >= 0) {
                kx[u] = k_pool[src[u]];
                vx[u] = v_pool[src[u]];
            }
#pragma unroll
        for (int u = 0; u < kWidenUnroll; ++u)
            if (src[u] >= 0) {
                wk[base + u * stride] = widen8<kBf16>(kx[u]);
                wv[base + u * stride] = widen8<false>(vx[u]);
            }
    }
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

}  // namespace
}  // namespace pkv

extern "C" size_t pkv_prefill_fp8_workspace_bytes(int num_seqs, int max_blocks_per_seq, int num_kv_heads,
                                                  int head_dim, int block_size) {
    if (num_seqs <= 0 || max_blocks_per_seq <= 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0) return 0;
    const size_t blocks = static_cast<size_t>(num_seqs) * max_blocks_per_seq;
    const size_t pool = blocks * num_kv_heads * block_size * head_dim * 2;
    return 2 * pkv::align256(pool) + pkv::align256(blocks * sizeof(int32_t));
}

extern "C" pkv_status pkv_paged_attn_prefill_fp8(void* out, const void* q, pkv_dtype q_dtype, const void* k_pool,
                                                 const void* v_pool, float k_scale, float v_scale,
                                                 const int32_t* block_tables, int max_blocks_per_seq,
                                                 const int32_t* context_lens, const int32_t* query_start,
                                                 int max_query_len, int num_seqs, int num_tokens, int num_heads,
                                                 int num_kv_heads, int head_dim, int block_size, int num_blocks,
                                                 float scale, void* workspace, size_t workspace_bytes,
                                                 uint32_t* device_error, void* stream) {
    using namespace pkv;
    PrefillLaunch p{};
    p.out = out;
    p.q = q;
    p.bf16 = q_dtype == PKV_BF16;
    p.v_f16 = true;
    p.k_pool = k_pool;
    p.v_pool = v_pool;
    p.k_tables = block_tables;
    p.max_blocks_per_seq = max_blocks_per_seq;
    p.context_lens = context_lens;
    p.query_start = query_start;
    p.max_query_len = max_query_len;
    p.num_seqs = num_seqs;
    p.num_tokens = num_tokens;
    p.num_heads = num_heads;
    p.num_kv_heads = num_kv_heads;
    p.head_dim = head_dim;
    p.block_size = block_size;
    p.num_blocks = num_blocks;
    p.scale = scale * k_scale;   // K is widened exactly; its scale joins the softmax scale
    p.v_mult_all = v_scale;      // V too; its scale multiplies the output rows
    p.err = device_error;
    p.stream = static_cast<cudaStream_t>(stream);
    // the checks of pkv_paged_attn_prefill, the scales first, before anything is launched
    if (!(scale > 0.f) || !std::isfinite(scale) || !(k_scale > 0.f) || !std::isfinite(k_scale) ||
        !(v_scale > 0.f) || !std::isfinite(v_scale) || !(p.scale > 0.f) || !std::isfinite(p.scale))
        return PKV_ERR_INVALID_ARG;
    const pkv_status chk = prefill_check(p, q_dtype == PKV_F16 || q_dtype == PKV_BF16);
    if (chk != PKV_OK || num_seqs == 0 || num_tokens == 0 || max_query_len == 0) return chk;
    const size_t need = pkv_prefill_fp8_workspace_bytes(num_seqs, max_blocks_per_seq, num_kv_heads, head_dim,
                                                        block_size);
    if (!workspace || workspace_bytes < need) return PKV_ERR_WORKSPACE;
    if (reinterpret_cast<uintptr_t>(workspace) & 255) return PKV_ERR_ALIGNMENT;

    const size_t blocks = static_cast<size_t>(num_seqs) * max_blocks_per_seq;
    const size_t pool = align256(blocks * num_kv_heads * block_size * head_dim * 2);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    void* wk = ws;
    void* wv = ws + pool;
    int32_t* wtab = reinterpret_cast<int32_t*>(ws + 2 * pool);
    // 8-byte units of an E4M3 block (head_dim 64 or 128: whole units)
    const long long units_per_block = static_cast<long long>(num_kv_heads) * block_size * head_dim / 8;
    const long long total = static_cast<long long>(blocks) * units_per_block;
    long long grid = (total + kWidenThreads - 1) / kWidenThreads;
    const long long cap = static_cast<long long>(num_sms()) * 8;
    if (grid > cap) grid = cap;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    auto launch = [&](auto kern) {
        return launch_pdl(kern, dim3(static_cast<unsigned>(grid)), dim3(kWidenThreads), 0, st,
                          static_cast<const uint2*>(k_pool), static_cast<const uint2*>(v_pool),
                          static_cast<uint4*>(wk), static_cast<uint4*>(wv), wtab, block_tables, context_lens, num_seqs,
                          max_blocks_per_seq, units_per_block, block_size, num_blocks, device_error);
    };
    const cudaError_t e = p.bf16 ? launch(widen_blocks_kernel<true>) : launch(widen_blocks_kernel<false>);
    if (e != cudaSuccess) return PKV_ERR_CUDA;
    p.k_pool = wk;
    p.v_pool = wv;
    p.k_tables = wtab;
    p.num_blocks = static_cast<int>(blocks);
    return prefill_launch(p);
}
