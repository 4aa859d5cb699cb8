// Host-side helpers shared by the launchers.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/pagedkv.h"

namespace pkv {

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// SM count and L2 size in bytes of the current device.
int num_sms();
long long l2_bytes();

// cuTensorMapEncodeTiled from the driver, looked up once through the runtime
// (no link-time dependency on libcuda).  nullptr if unavailable.
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn encode_tiled_fn();

// One launch of the tensor-core prefill kernel (prefill.cu), for the 16-bit entry point and for
// the E4M3 one after its widening pass.
struct PrefillLaunch {
    void* out;
    const void* q;
    bool bf16;                 // q, K and out are bf16 (else f16)
    bool v_f16;                // V is f16 (an f16 cache, or narrowed / widened): one f16 P.V product;
                               // else (bf16 V) the weights enter as a high and a low bf16 part
    const void* k_pool;
    const void* v_pool;
    const int32_t* k_tables;
    const int32_t* v_tables;   // null: V blocks through k_tables
    int max_blocks_per_seq;
    const int32_t* context_lens;
    const int32_t* query_start;
    int max_query_len, num_seqs, num_tokens, num_heads, num_kv_heads, head_dim, block_size;
    int num_blocks;            // of the K pool (and of the V pool when v_tables is null)
    int v_num_blocks;          // of the V pool when v_tables is set
    float scale;
    const float* v_mult;       // per (sequence, KV head) factor of the output, or null
    float v_mult_all;          // factor of every output row
    uint32_t* err;
    cudaStream_t stream;
};

// The host-side checks of a prefill call (sizes, supported shapes, pointers, alignment), in the
// order the entry points report them; PKV_OK also for an empty call.
pkv_status prefill_check(const PrefillLaunch& p, bool dtype_supported);
pkv_status prefill_launch(const PrefillLaunch& p);

// Launch with programmatic stream serialisation: the kernel may begin while the
// previous kernel on the stream drains (it synchronises itself with pdl_wait()).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                       Args&&... args) {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, static_cast<Args&&>(args)...);
}

}  // namespace pkv
