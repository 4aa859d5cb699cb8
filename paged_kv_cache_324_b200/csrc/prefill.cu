// Chunked prefill over the paged KV cache on the 5th-generation tensor cores.
//
// Every query of a chunk attends causally to the cached tokens up to its own
// position (Wikipedia "PagedAttention", section "Mathematical formulation",
// token form, for each query position of the chunk); unlike decode this is a
// dense contraction ("vLLM and PagedAttention" transcript, opening paragraph:
// prefill maps onto large matrix products), so both products run as
// tcgen05.mma with the accumulators in tensor memory.
//
// One CTA = two tiles of 128 query rows (tile A, then tile B: 128 / G tokens
// each, x the G query heads of one KV head) of one sequence, against 128-key
// tiles of that KV head read through the block table.  Both query tiles use
// every K/V tile the CTA loads, which halves the K/V bytes per FLOP of a
// one-tile CTA.  Warp roles (19 warps):
//   warps 0,18 TMA: warp 0 both Q tiles once, then K tiles, warp 18 V tiles,
//              each into a 2-stage ring, block by block (one 4-D box per 16-
//              or 32-token block and 64-column chunk, 128-byte swizzle), each
//              reading its table entries one tile ahead;
//   warp 1     allocates all 512 TMEM columns (S_A, S_B, O_A, O_B); one thread
//              issues the MMAs in the order
//                S_A(0), PV_A(0), S_A(1), S_B(0), PV_B(0), S_B(1), PV_A(1), S_A(2), ...
//              (tile B half a period behind tile A)
//              S = Q K^T (M=128, N=128, both operands K-major in shared
//              memory) and O += P V (M=128, N=head_dim; P read from tensor
//              memory, V an MN-major shared-memory operand; for bf16 a second
//              product O += P_lo V over the same V tile).  The MMAs of a CTA
//              execute in issue order, which is what lets P overwrite the S it
//              came from and S_X(j+1) overwrite P_X(j) once PV_X(j) has read it;
//   warps 2-9  softmax of tile A, warps 10-17 of tile B, two warps per TMEM
//              lane quarter: each thread takes one query row (TMEM lane = row)
//              and 64 of its 128 keys, the two halves of a row exchanging their
//              maxima through shared memory.  Read S, mask, online softmax in
//              base 2 with a running maximum that is only moved when the new
//              one exceeds it by more than 2^8 (the result does not depend on
//              the reference maximum; the lag only bounds the weights), write P
//              as packed f16 pairs into the upper half of the same S columns
//              with tcgen05.st (for a bf16 V: bf16 P, and the residual
//              P - bf16(P) into the lower half, so that P.V sees ~16
//              significant bits of every weight), and rescale O in TMEM when
//              the maximum moves; finally O * f / l (f: V's scale), written into the
//              query tile's own shared memory (free by then) and sent out by
//              warp 0 with one TMA store per 64-column chunk, so that whole
//              128-byte rows reach HBM (a tile cut short by the chunk's end is
//              stored row by row instead).
// While tile A's softmax works on S_A(j+1), the tensor core computes PV_B(j)
// and S_B(j+1), and the other way round.
//
// A bf16 cache's V is normally narrowed to f16 before this kernel runs (two small passes below,
// each (sequence, KV head) scaled by its own power of two), so that P enters P.V as one f16
// operand with 11 significant bits: that keeps the weights' rounding inside the attention
// tolerance with one product per key tile instead of the two the bf16 split needs.
//
// Keys beyond the last one any row of the CTA needs are never loaded; their V
// rows are zeroed in shared memory (their weights are exactly 0, but 0 times
// stale bytes could be NaN).  Every wait is bounded; a wait that gives up
// sets PKV_DEVERR_TIMEOUT, the other roles stop at their next wait, in-flight
// copies and MMAs are drained (bounded) and TMEM is freed before exit.

#include <cmath>
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "pkv_device.cuh"
#include "pkv_host.h"

namespace pkv {
namespace {

constexpr int kRows = 128;            // query rows per tile: MMA M, one TMEM lane each
constexpr int kTiles = 2;             // query tiles per CTA
constexpr int kKeys = 128;            // keys per K/V tile: N of S = Q K^T, K of O += P V
constexpr int kKStages = 2;
constexpr int kVStages = 2;
constexpr int kHalves = 2;            // softmax warps per TMEM lane quarter and tile: each takes 64 of 128 keys
constexpr int kTileWarps = 4 * kHalves;
constexpr int kVWarp = 2 + kTiles * kTileWarps;
constexpr int kPThreads = 32 * (kVWarp + 1);   // warp 0 TMA (Q, K), warp 1 MMA, softmax, last warp TMA (V)
constexpr uint32_t kTmemCols = 512;   // S_A [0,128), S_B [128,256), O_A [256,384), O_B [384,512)
// P_X: the upper half of S_X, packed pairs; for bf16 the residual P_X - bf16(P_X) (P_lo) goes over the
// lower half, so that the P.V product sees ~16 significant bits of each weight (two MMAs per key step)
constexpr uint32_t kTmemS = 0, kTmemO = 256, kTmemP = 64, kTmemPlo = 0;
constexpr float kMaxLag = 8.0f;       // log2 of the largest weight the lagging maximum allows
constexpr uint32_t kChunkBytes = kRows * 128;   // 128 rows x 128 bytes: one 64-column chunk

template <int D>
struct PGeo {
    static constexpr int kChunks = D / 64;
    static constexpr uint32_t kTile = kChunks * kChunkBytes;   // one Q tile, or one K or V stage
    static constexpr uint32_t kQ = 0;
    static constexpr uint32_t kK = kQ + kTiles * kTile;
    static constexpr uint32_t kV = kK + kKStages * kTile;
    static constexpr uint32_t kEnd = kV + kVStages * kTile;
    // +1 KB to align the base; at least 120 KB so that one CTA holds an SM (TMEM is not shared)
    static constexpr uint32_t kSmemBytes = (kEnd + 1024 > 120u * 1024u) ? kEnd + 1024 : 120u * 1024u;
};

struct PrefillArgs {
    void* out;
    const int32_t* block_tables;   // K blocks
    const int32_t* v_tables;       // V blocks (the same table, or a workspace pool's own)
    const int32_t* context_lens;
    const int32_t* query_start;
    const float* v_mult;           // per (sequence, KV head) factor of the output, or null
    uint32_t* err;
    int max_blocks_per_seq;
    int num_tokens;
    int num_heads;
    int num_blocks;                // of the K pool
    int v_num_blocks;              // of the V pool
    int group;                     // G = num_heads / num_kv_heads
    float scale_log2;              // scale * log2(e)
    float v_mult_all;              // factor of every output row (an E4M3 cache's V scale, else 1)
};

// ---- tcgen05 / TMEM primitives (inline PTX) ---------------------------------------

__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Shared-memory matrix descriptor, 128-byte swizzle, sm_100 version field.
// lbo/sbo in bytes: K-major tiles use sbo = 1024 (8-row groups of 128-byte rows);
// MN-major tiles add lbo = the distance between 64-element column chunks.
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
    return static_cast<uint64_t>((addr & 0x3FFFFu) >> 4) |
           (static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16) |
           (static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32) |
           (1ull << 46) |          // descriptor version for sm_100
           (2ull << 61);           // SWIZZLE_128B
}

// Instruction descriptor of kind::f16: f32 accumulator, A and B of one 16-bit type,
// A K-major, B K-major or MN-major, shape M x N.
__host__ __device__ constexpr uint32_t mma_idesc(bool bf16, bool b_mn_major, int M, int N) {
    return (1u << 4) | ((bf16 ? 1u : 0u) << 7) | ((bf16 ? 1u : 0u) << 10) | ((b_mn_major ? 1u : 0u) << 16) |
           (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}

__device__ __forceinline__ void mma_f16(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc, bool accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a), "l"(b), "r"(idesc), "r"(accumulate ? 1u : 0u)
        : "memory");
}

// The same with A read from tensor memory (lane = row, two 16-bit K elements per column).
__device__ __forceinline__ void mma_f16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b, uint32_t idesc,
                                           bool accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b), "r"(idesc), "r"(accumulate ? 1u : 0u)
        : "memory");
}

// Arrive once on `bar` when every MMA this thread issued so far has completed.
__device__ __forceinline__ void mma_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                 : "memory");
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
        "%14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
}

// tcgen05.ld delivers its registers asynchronously: the wait takes them as operands so
// that no use of them can be scheduled before it.
__device__ __forceinline__ void tmem_ld32_wait(uint32_t taddr, uint32_t (&r)[32]) {
    tmem_ld32(taddr, r);
    asm volatile(
        "tcgen05.wait::ld.sync.aligned;"
        : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
          "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15]),
          "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]), "+r"(r[22]), "+r"(r[23]),
          "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]), "+r"(r[29]), "+r"(r[30]), "+r"(r[31])
        :
        : "memory");
}

__device__ __forceinline__ void tmem_ld64_wait(uint32_t taddr, uint32_t (&r)[64]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x64.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32, %33, %34, %35, %36, %37, %38, %39, %40, %41, %42, %43, %44, %45, %46, %47, %48, %49, %50, %51, %52, %53, %54, %55, %56, %57, %58, %59, %60, %61, %62, %63}, [%64];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31]),
          "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]), "=r"(r[37]), "=r"(r[38]), "=r"(r[39]),
          "=r"(r[40]), "=r"(r[41]), "=r"(r[42]), "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]),
          "=r"(r[48]), "=r"(r[49]), "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]),
          "=r"(r[56]), "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]), "=r"(r[62]), "=r"(r[63])
        : "r"(taddr));
    asm volatile(
        "tcgen05.wait::ld.sync.aligned;"
        : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
          "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15]),
          "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]), "+r"(r[22]), "+r"(r[23]),
          "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]), "+r"(r[29]), "+r"(r[30]), "+r"(r[31]),
          "+r"(r[32]), "+r"(r[33]), "+r"(r[34]), "+r"(r[35]), "+r"(r[36]), "+r"(r[37]), "+r"(r[38]), "+r"(r[39]),
          "+r"(r[40]), "+r"(r[41]), "+r"(r[42]), "+r"(r[43]), "+r"(r[44]), "+r"(r[45]), "+r"(r[46]), "+r"(r[47]),
          "+r"(r[48]), "+r"(r[49]), "+r"(r[50]), "+r"(r[51]), "+r"(r[52]), "+r"(r[53]), "+r"(r[54]), "+r"(r[55]),
          "+r"(r[56]), "+r"(r[57]), "+r"(r[58]), "+r"(r[59]), "+r"(r[60]), "+r"(r[61]), "+r"(r[62]), "+r"(r[63])
        :
        : "memory");
}

// Paired fp32 arithmetic (one instruction for two lanes of work) and a three-input maximum.
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {
    float2 d;
    asm("{.reg .b64 pa, pb, pc, pd;\n\t"
        "mov.b64 pa, {%2, %3};\n\tmov.b64 pb, {%4, %5};\n\tmov.b64 pc, {%6, %7};\n\t"
        "fma.rn.f32x2 pd, pa, pb, pc;\n\tmov.b64 {%0, %1}, pd;}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
    return d;
}
__device__ __forceinline__ float2 add2(float2 a, float2 b) {
    float2 d;
    asm("{.reg .b64 pa, pb, pd;\n\t"
        "mov.b64 pa, {%2, %3};\n\tmov.b64 pb, {%4, %5};\n\t"
        "add.rn.f32x2 pd, pa, pb;\n\tmov.b64 {%0, %1}, pd;}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}
__device__ __forceinline__ float2 sub2(float2 a, float2 b) {
    float2 d;
    asm("{.reg .b64 pa, pb, pd;\n\t"
        "mov.b64 pa, {%2, %3};\n\tmov.b64 pb, {%4, %5};\n\t"
        "sub.rn.f32x2 pd, pa, pb;\n\tmov.b64 {%0, %1}, pd;}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}
__device__ __forceinline__ float max3f(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

// 2^x with the multi-function unit's approximation (subnormal results flush to zero).
__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
        "%14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
        "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]),
        "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]),
        "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
}

__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t (&r)[8]) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(taddr),
                 "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
                 : "memory");
}

__device__ __forceinline__ void tmem_st4(uint32_t taddr, const uint32_t (&r)[4]) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x4.b32 [%0], {%1, %2, %3, %4};" ::"r"(taddr), "r"(r[0]), "r"(r[1]),
                 "r"(r[2]), "r"(r[3])
                 : "memory");
}

__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* map, uint32_t bar, int c0, int c1,
                                            int c2) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(bar)
        : "memory");
}

// Shared memory -> global through a tensor map (bulk-group completion).
__device__ __forceinline__ void tma_store_3d(const CUtensorMap* map, uint32_t src, int c0, int c1, int c2) {
    asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.tile.bulk_group [%0, {%1, %2, %3}], [%4];" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(c0), "r"(c1), "r"(c2), "r"(src)
                 : "memory");
}

__device__ __forceinline__ uint64_t l2_policy_evict_last() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
    return p;
}

__device__ __forceinline__ void sts128(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
    asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d)
                 : "memory");
}

template <bool kBf16>
__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
    if constexpr (kBf16) {
        __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
        return *reinterpret_cast<uint32_t*>(&v);
    } else {
        __half2 v = __floats2half2_rn(lo, hi);
        return *reinterpret_cast<uint32_t*>(&v);
    }
}

// Shared flags of a CTA: a wait gave up (every role stops), a block id was bad.
struct CtaFlags {
    int abort;
    int bad;
    uint32_t tmem_base;
    float vmul;           // the factor of this CTA's output rows (V's scale)
};

// Bounded wait that also stops when another role of the CTA already gave up.
__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, CtaFlags* f, uint32_t* err) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t end = global_timer_ns() + kWaitLimitNs;
    while (true) {
#pragma unroll 1
        for (int i = 0; i < 32; ++i)
            if (mbar_try_wait(bar, parity)) return true;
        if (*reinterpret_cast<volatile int*>(&f->abort)) return false;
        if (global_timer_ns() > end) {
            raise_error(err, PKV_DEVERR_TIMEOUT);
            *reinterpret_cast<volatile int*>(&f->abort) = 1;
            return false;
        }
    }
}

// Same, decided once for a whole warp (every lane waits; all continue only if all succeeded).
__device__ __forceinline__ bool warp_wait_bar(uint32_t bar, uint32_t parity, CtaFlags* f, uint32_t* err) {
    const bool ok = wait_bar(bar, parity, f, err);
    return __all_sync(0xffffffffu, ok);
}

// kBf16: q, K and the output are bf16 (else f16).  kSplitP (bf16 only): V is bf16 too and the
// weights enter P.V as a high and a low bf16 part; otherwise V is f16 (an f16 cache, or V narrowed
// or widened to f16 with its scale applied to the output) and P is one f16 operand.
template <int D, int BS, bool kBf16, bool kSplitP>
__global__ void __launch_bounds__(kPThreads, 1)
paged_prefill_kernel(const PrefillArgs a, const __grid_constant__ CUtensorMap qmap,
                     const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap,
                     const __grid_constant__ CUtensorMap omap) {
    using Gm = PGeo<D>;
    static_assert(kBf16 || !kSplitP, "the two-part weights are for bf16 V");
    constexpr bool kPvBf16 = kSplitP;                // the type of P and V in O += P V
    constexpr int kTB = kKeys / BS;                  // blocks per key tile
    constexpr uint32_t kBoxBytes = BS * 128;         // one block x one 64-column chunk
    extern __shared__ uint8_t smem_raw[];
    __shared__ __align__(8) uint64_t bars[2 * kKStages + 2 * kVStages + 8 + kTiles * 4];
    __shared__ CtaFlags flags;
    __shared__ float red[2][kTiles][kHalves][kRows];   // [tile parity][query tile][half][row]: partial maxima

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = a.group, TQ = kRows / G;           // tokens per query tile
    const int kvh = blockIdx.y, s = blockIdx.z;

    pdl_wait();   // q, the pool and the tables may come from the previous kernel on the stream
    const int q0 = __ldg(a.query_start + s), q1 = __ldg(a.query_start + s + 1);
    const int L = __ldg(a.context_lens + s);
    if (q0 < 0 || q1 < q0 || q1 > a.num_tokens) {        // rows of unknown place: nothing to write
        if (threadIdx.x == 0 && blockIdx.x == 0) raise_error(a.err, PKV_DEVERR_CONTEXT_LEN);
        return;
    }
    const int C = q1 - q0;
    const int ncta = (C + kTiles * TQ - 1) / (kTiles * TQ);
    if (blockIdx.x == 0 && threadIdx.x == 0 && ncta > static_cast<int>(gridDim.x))
        raise_error(a.err, PKV_DEVERR_CONTEXT_LEN);      // longer than max_query_len: rows left unwritten
    if (static_cast<int>(blockIdx.x) >= ncta) return;
    if (grid_timed_out(a.err)) return;   // a wait elsewhere gave up: finish at once
    const int t0 = (ncta - 1 - static_cast<int>(blockIdx.x)) * kTiles * TQ;   // longest tiles first
    const int rows_cta = min(kTiles * TQ, C - t0);                              // tokens of this CTA

    if (C > L || L > a.max_blocks_per_seq * BS) {         // positions undefined: NaN rows
        if (threadIdx.x == 0) raise_error(a.err, PKV_DEVERR_CONTEXT_LEN);
        for (int i = threadIdx.x; i < rows_cta * G * D; i += kPThreads) {
            const int t = i / (G * D), rem = i % (G * D);
            const size_t o = (static_cast<size_t>(q0 + t0 + t) * a.num_heads + kvh * G) * D + rem;
            reinterpret_cast<uint16_t*>(a.out)[o] = kBf16 ? 0x7FC0u : 0x7E00u;
        }
        return;
    }
    const bool has_b = rows_cta > TQ;
    // last key each tile's rows attend; key tiles each tile needs; the CTA loads the larger range
    const int pq_max_a = min(L - C + t0 + TQ - 1, L - 1);
    const int pq_max_b = min(L - C + t0 + 2 * TQ - 1, L - 1);
    const int ntk_a = pq_max_a / kKeys + 1;
    const int ntk_b = has_b ? pq_max_b / kKeys + 1 : 0;
    const int ntk = max(ntk_a, ntk_b);
    const int pq_max = has_b ? pq_max_b : pq_max_a;
    const int nblk = (pq_max + 1 + BS - 1) / BS;           // blocks holding keys 0..pq_max

    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_addr(smem);
    const uint32_t sQ = sbase + Gm::kQ, sK = sbase + Gm::kK, sV = sbase + Gm::kV;
    const uint32_t b0 = smem_addr(bars);
    auto k_full = [&](int i) { return b0 + 8u * i; };
    auto k_empty = [&](int i) { return b0 + 8u * (kKStages + i); };
    auto v_full = [&](int i) { return b0 + 8u * (2 * kKStages + i); };
    auto v_empty = [&](int i) { return b0 + 8u * (2 * kKStages + kVStages + i); };
    const uint32_t bar_q = b0 + 8u * (2 * kKStages + 2 * kVStages);
    auto s_full = [&](int t) { return bar_q + 8u * (1 + t); };    // per query tile
    auto p_full = [&](int t) { return bar_q + 8u * (3 + t); };
    auto o_done = [&](int t) { return bar_q + 8u * (5 + t); };    // the tile's last P.V product completed
    const uint32_t drain = bar_q + 8u * 7;
    auto xchg = [&](int t, int quarter) { return bar_q + 8u * (8 + t * 4 + quarter); };   // the halves of a row

    if (threadIdx.x == 0) {
        for (int i = 0; i < kKStages; ++i) {
            mbar_init(k_full(i), 1);
            mbar_init(k_empty(i), 1);
        }
        for (int i = 0; i < kVStages; ++i) {
            mbar_init(v_full(i), 1);
            mbar_init(v_empty(i), 1);
        }
        mbar_init(bar_q, 1);
        for (int t = 0; t < kTiles; ++t) {
            mbar_init(s_full(t), 1);
            mbar_init(p_full(t), kTileWarps);
            mbar_init(o_done(t), 1);
            for (int q = 0; q < 4; ++q) mbar_init(xchg(t, q), kHalves);
        }
        mbar_init(drain, 1);
        flags.abort = 0;
        flags.bad = 0;
        mbar_fence_init();
        // both Q tiles are requested at once, so that their load overlaps the TMEM allocation and
        // the CTA-wide barrier below
        tma_prefetch_desc(&qmap);
        mbar_arrive_expect_tx(bar_q, kTiles * Gm::kTile);
#pragma unroll
        for (int t = 0; t < kTiles; ++t)
#pragma unroll
            for (int c = 0; c < Gm::kChunks; ++c)
                tma_load_3d(sQ + t * Gm::kTile + c * kChunkBytes, &qmap, bar_q, c * 64, kvh * G, q0 + t0 + t * TQ);
        flags.vmul = a.v_mult_all * (a.v_mult ? __ldg(a.v_mult + static_cast<size_t>(s) * gridDim.y + kvh) : 1.f);
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_addr(&flags.tmem_base)),
                     "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = flags.tmem_base;

    if (warp == 0 || warp == kVWarp) {
        // ---------------- TMA producers: warp 0 loads Q and K, the last warp loads V ----------------
        const bool is_k = warp == 0;
        const int nst = is_k ? kKStages : kVStages;
        const uint64_t pol = l2_policy_evict_last();      // K/V tiles are read again by the other query tiles
        if (is_k && lane == 0) {
            tma_prefetch_desc(&kmap);
            tma_prefetch_desc(&vmap);
        }
        const CUtensorMap* map = is_k ? &kmap : &vmap;
        const uint32_t ring = is_k ? sK : sV;
        const int32_t* trow = (is_k ? a.block_tables : a.v_tables) + static_cast<size_t>(s) * a.max_blocks_per_seq;
        const int nblocks = is_k ? a.num_blocks : a.v_num_blocks;
        int issued = 0;                                   // tiles whose copies were issued
        // table entries are read one tile ahead so that their latency hides behind the copies
        int pid_next = (lane < kTB && lane < nblk) ? __ldg(trow + lane) : -1;
        for (int j = 0; j < ntk; ++j) {
            const int pid = pid_next;
            const int nb = (j + 1) * kTB + lane;
            pid_next = (j + 1 < ntk && lane < kTB && nb < nblk) ? __ldg(trow + nb) : -1;
            const bool want = lane < kTB && j * kTB + lane < nblk;
            const bool bad = want && (pid < 0 || pid >= nblocks);
            const unsigned ok_mask = __ballot_sync(0xffffffffu, want && !bad);
            if (__any_sync(0xffffffffu, bad) && lane == 0) {
                raise_error(a.err, PKV_DEVERR_BLOCK_ID);
                flags.bad = 1;
            }
            const uint32_t bytes = __popc(ok_mask) * kBoxBytes * Gm::kChunks;
            const int st = j % nst;
            const uint32_t full = is_k ? k_full(st) : v_full(st), empty = is_k ? k_empty(st) : v_empty(st);
            if (j >= nst && !warp_wait_bar(empty, ((j / nst) - 1) & 1, &flags, a.err)) break;
            if (lane == 0) mbar_arrive_expect_tx(full, bytes);
            issued = j + 1;
            for (int b = 0; b < kTB; ++b) {
                const int p = __shfl_sync(0xffffffffu, pid, b);
                if (lane == 0 && ((ok_mask >> b) & 1u)) {
#pragma unroll
                    for (int c = 0; c < Gm::kChunks; ++c)
                        tma_load_4d(ring + st * Gm::kTile + c * kChunkBytes + b * kBoxBytes, map, full, c * 64, 0, kvh,
                                    p, pol);
                }
            }
        }
        // drain: the last copies of each stage must land before the CTA may exit
        if (lane == 0) {
            const uint64_t end = global_timer_ns() + kWaitLimitNs;
            if (is_k) mbar_wait(bar_q, 0, end);
            for (int j = max(0, issued - nst); j < issued; ++j)
                mbar_wait(is_k ? k_full(j % nst) : v_full(j % nst), (j / nst) & 1, end);
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer (one thread) ----------------
        if (lane == 0) {
            constexpr uint32_t idesc_s = mma_idesc(kBf16, false, kRows, kKeys);
            constexpr uint32_t idesc_o = mma_idesc(kPvBf16, true, kRows, D);
            int k_waited = -1;                            // the last key tile whose arrival was awaited
            auto issue_s = [&](int t, int j) -> bool {    // S_t(j) = Q_t K_j^T into S_t
                const int ks = j % kKStages;
                if (k_waited < j) {
                    if (!wait_bar(k_full(ks), (j / kKStages) & 1, &flags, a.err)) return false;
                    k_waited = j;
                }
                tc_fence_after();
#pragma unroll
                for (int k = 0; k < D / 16; ++k) {
                    const uint32_t off = (k >> 2) * kChunkBytes + (k & 3) * 32;
                    mma_f16(tmem + kTmemS + t * kKeys, smem_desc(sQ + t * Gm::kTile + off, 16, 1024),
                            smem_desc(sK + ks * Gm::kTile + off, 16, 1024), idesc_s, k > 0);
                }
                mma_commit(s_full(t));
                return true;
            };
            auto issue_pv = [&](int t, int j) -> bool {   // O_t += P_t V_j, P_t from tensor memory
                if (!wait_bar(p_full(t), j & 1, &flags, a.err)) return false;
                tc_fence_after();
                const int vs = j % kVStages;
#pragma unroll
                for (int kk = 0; kk < kKeys / 16; ++kk) {
                    const uint64_t vdesc = smem_desc(sV + vs * Gm::kTile + kk * 16 * 128, kChunkBytes, 1024);
                    mma_f16_ts(tmem + kTmemO + t * 128, tmem + kTmemS + t * kKeys + kTmemP + kk * 8, vdesc, idesc_o,
                               j > 0 || kk > 0);
                    if constexpr (kSplitP)   // the weights' bf16 residual against the same V rows
                        mma_f16_ts(tmem + kTmemO + t * 128, tmem + kTmemS + t * kKeys + kTmemPlo + kk * 8, vdesc,
                                   idesc_o, true);
                }
                if (j == (t == 0 ? ntk_a : ntk_b) - 1) mma_commit(o_done(t));
                return true;
            };
            int v_waited = -1;
            auto pv_then_s = [&](int t, int j) -> bool {   // PV_t(j), then S_t(j+1) over the P it read
                if (v_waited < j) {
                    if (!wait_bar(v_full(j % kVStages), (j / kVStages) & 1, &flags, a.err)) return false;
                    v_waited = j;
                }
                if (!issue_pv(t, j)) return false;
                return j + 1 < (t == 0 ? ntk_a : ntk_b) ? issue_s(t, j + 1) : true;
            };
            // Tile B runs half a period behind tile A, so that each tile's softmax overlaps the other
            // tile's P.V and S products: S_A(0), PV_A(0) S_A(1), S_B(0), then for each j
            // PV_B(j) S_B(j+1), PV_A(j+1) S_A(j+2).
            bool ok = wait_bar(bar_q, 0, &flags, a.err);
            if (ok) ok = issue_s(0, 0);
            if (ok) ok = pv_then_s(0, 0);
            if (ok && has_b) ok = issue_s(1, 0);
            if (ok) mma_commit(k_empty(0));
            for (int j = 0; ok && j < ntk; ++j) {
                if (has_b && j < ntk_b) ok = pv_then_s(1, j);
                if (!ok) break;
                mma_commit(v_empty(j % kVStages));                   // V_j: PV_A(j) and PV_B(j) issued
                if (j + 1 < ntk) mma_commit(k_empty((j + 1) % kKStages));   // K_{j+1}: both S issued
                if (j + 1 < ntk_a) ok = pv_then_s(0, j + 1);
            }
            // drain: every MMA issued so far completes before TMEM is freed
            mma_commit(drain);
            mbar_wait(drain, 0, global_timer_ns() + kWaitLimitNs);
        }
        __syncwarp();
    } else {
        // ---------------- softmax: row = TMEM lane, half = which 64 of the row's keys ----------------
        const int t = (warp - 2) / kTileWarps;
        const int half = ((warp - 2) % kTileWarps) >> 2;
        const int quarter = warp & 3;
        const int row = quarter * 32 + lane;
        const uint32_t tl = tmem + (static_cast<uint32_t>(quarter * 32) << 16);   // this warp's lanes
        const uint32_t tS = tl + kTmemS + t * kKeys, tO = tl + kTmemO + t * 128;
        constexpr int kOCols = D / kHalves;                // O columns this thread rescales and stores
        const int tq = t * TQ + row / G;                  // token of this row within the CTA
        const int pq = min(L - C + t0 + tq, L - 1);
        const int my_ntk = t == 0 ? ntk_a : ntk_b;
        float m_used = -INFINITY, l = 0.f;
        bool ok = true;
        for (int j = 0; j < my_ntk; ++j) {
            // S_t(j) complete means PV_t(j-1) has completed too (issue order): P and O are free
            if (!warp_wait_bar(s_full(t), j & 1, &flags, a.err)) { ok = false; break; }
            tc_fence_after();
            const int kbase = j * kKeys + half * 64;
            const bool mask = kbase + 63 > pq;
            float x[64];
            {
                uint32_t r[64];
                tmem_ld64_wait(tS + half * 64, r);
                if (mask) {                                   // only tiles that cross this row's position
#pragma unroll
                    for (int i = 0; i < 64; ++i) x[i] = kbase + i > pq ? -INFINITY : __uint_as_float(r[i]);
                } else {
#pragma unroll
                    for (int i = 0; i < 64; ++i) x[i] = __uint_as_float(r[i]);
                }
            }
            float mp[8];                                      // eight chains of three-input maxima, then a tree
#pragma unroll
            for (int i = 0; i < 8; ++i)
                mp[i] = fmaxf(max3f(max3f(x[i], x[i + 8], x[i + 16]), x[i + 24], x[i + 32]),
                              max3f(x[i + 40], x[i + 48], x[i + 56]));
            float mx = max3f(max3f(mp[0], mp[1], mp[2]), max3f(mp[3], mp[4], mp[5]), fmaxf(mp[6], mp[7]));
            // the row's maximum over both halves; after this exchange both halves have read their S,
            // so P may be written over the S columns of keys 64-127
            red[j & 1][t][half][row] = mx;
            __syncwarp();
            if (lane == 0) mbar_arrive(xchg(t, quarter));
            if (!warp_wait_bar(xchg(t, quarter), j & 1, &flags, a.err)) { ok = false; break; }
            mx = fmaxf(mx, red[j & 1][t][half ^ 1][row]);
            const float m_cand = mx * a.scale_log2;
            const bool move = m_cand > m_used + kMaxLag;
            float alpha = 1.f;
            if (move) {
                alpha = ex2(m_used - m_cand);
                m_used = m_cand;
            }
            const float2 sc2 = make_float2(a.scale_log2, a.scale_log2), nm2 = make_float2(-m_used, -m_used);
            float2 sp[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
            for (int h = 0; h < 8; ++h) {                    // 8 keys (4 packed words) at a time
                uint32_t pk[4], pl[4];
#pragma unroll
                for (int c = 0; c < 8; c += 2) {
                    const float2 e = fma2(make_float2(x[8 * h + c], x[8 * h + c + 1]), sc2, nm2);
                    const float2 p = make_float2(ex2(e.x), ex2(e.y));
                    sp[(c >> 1) & 1] = add2(sp[(c >> 1) & 1], p);
                    pk[c / 2] = pack2<kPvBf16>(p.x, p.y);
                    if constexpr (kSplitP) {
                        // p - bf16(p) is exact in fp32; widening bf16 is a 16-bit shift
                        const float2 r = sub2(p, make_float2(__uint_as_float(pk[c / 2] << 16),
                                                             __uint_as_float(pk[c / 2] & 0xffff0000u)));
                        pl[c / 2] = pack2<true>(r.x, r.y);
                    }
                }
                tmem_st4(tS + kTmemP + half * 32 + h * 4, pk);
                if constexpr (kSplitP) tmem_st4(tS + kTmemPlo + half * 32 + h * 4, pl);
            }
            const float2 s01 = add2(sp[0], sp[1]);
            l = l * alpha + (s01.x + s01.y);
            if (j > 0 && __any_sync(0xffffffffu, move)) {
#pragma unroll
                for (int c = 0; c < kOCols / 32; ++c) {
                    uint32_t r[32];
                    tmem_ld32_wait(tO + half * kOCols + c * 32, r);
#pragma unroll
                    for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
                    tmem_st32(tO + half * kOCols + c * 32, r);
                }
            }
            tmem_wait_st();
            if (j == ntk - 1 && j * kKeys + kKeys - 1 > pq_max) {
                // keys past pq_max were not loaded (or are unwritten slots): zero their V rows (each half its
                // 64-column chunk).  When both query tiles reach this tile they write the same zeros.
                const int vs = j % kVStages;
                if (!warp_wait_bar(v_full(vs), (j / kVStages) & 1, &flags, a.err)) { ok = false; break; }
                if (half < Gm::kChunks && j * kKeys + row > pq_max) {
#pragma unroll
                    for (int u = 0; u < 8; ++u)
                        sts128(sV + vs * Gm::kTile + half * kChunkBytes + row * 128 + ((u ^ (row & 7)) << 4), 0u, 0u,
                               0u, 0u);
                }
                fence_proxy_async_smem();
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(p_full(t));
        }
        if (ok && my_ntk > 0) ok = warp_wait_bar(o_done(t), 0, &flags, a.err);
        pdl_trigger();
        // partial row sums: the parity buffer the last exchange did not use is free by now
        // the output factor (V's scale) divides the row sum, so that 1 / sum brings it in
        red[my_ntk & 1][t][half][row] = l / flags.vmul;
        // the output is written after the CTA-wide barrier below, which also publishes flags.bad
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        // every lane takes part in the warp-wide TMEM loads; only rows of the chunk are stored
        const bool live = tq < rows_cta;
        const bool aborted = *reinterpret_cast<volatile int*>(&flags.abort) != 0;
        const bool nan_out = !ok || flags.bad || aborted;
        // a query tile with all TQ tokens goes through its Q tile's shared memory (free now: the
        // last S product that read it has completed) and one TMA store per 64-column chunk, so
        // that whole 128-byte rows reach HBM; a partial tile (or a CTA that gave up a wait, whose
        // copies may not have landed) stores its rows directly
        const bool staged = (t + 1) * TQ <= rows_cta && !aborted;
        uint16_t* orow = reinterpret_cast<uint16_t*>(a.out) +
                         (static_cast<size_t>(q0 + t0 + (live ? tq : 0)) * a.num_heads + kvh * G + row % G) * D +
                         half * kOCols;
        uint8_t* srow_g = smem + Gm::kQ + t * Gm::kTile + row * 128;   // this row of the Q tile (generic)
        const float inv = 1.f / (red[my_ntk & 1][t][0][row] + red[my_ntk & 1][t][1][row]);
#pragma unroll
        for (int c = 0; c < kOCols / 32; ++c) {
            uint32_t r[32];
            tmem_ld32_wait(tO + half * kOCols + c * 32, r);
            if (live) {
                uint32_t w[16];
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    w[i] = nan_out ? (kBf16 ? 0x7FC07FC0u : 0x7E007E00u)
                                   : pack2<kBf16>(__uint_as_float(r[2 * i]) * inv, __uint_as_float(r[2 * i + 1]) * inv);
                // staged: 16-byte units of the 64-column chunk in the 128-byte swizzle the Q tile was
                // loaded with (row = TMEM lane: token-major, head-minor); else the row in global memory
                const int col = half * kOCols + c * 32;
                uint8_t* sbase_c = srow_g + (col / 64) * kChunkBytes;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    uint4* dst = staged ? reinterpret_cast<uint4*>(sbase_c + ((((col % 64) / 8 + i) ^ (row & 7)) << 4))
                                        : reinterpret_cast<uint4*>(orow + c * 32) + i;
                    *dst = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
                }
            }
        }
        fence_proxy_async_smem();   // the staged rows become visible to the TMA store
        tc_fence_before();
        __syncthreads();
        return;   // warp 1 frees TMEM after the second barrier, warp 0 stores the staged tiles
    }
    // producer and MMA warps: meet the softmax warps at both barriers
    pdl_trigger();
    tc_fence_before();
    __syncthreads();
    __syncthreads();
    tc_fence_after();
    if (warp == 0 && lane == 0 && !*reinterpret_cast<volatile int*>(&flags.abort)) {
        int stores = 0;
#pragma unroll
        for (int t = 0; t < kTiles; ++t)
            if ((t + 1) * TQ <= rows_cta) {
#pragma unroll
                for (int c = 0; c < Gm::kChunks; ++c)
                    tma_store_3d(&omap, sQ + t * Gm::kTile + c * kChunkBytes, c * 64, kvh * G, q0 + t0 + t * TQ);
                ++stores;
            }
        if (stores) {
            asm volatile("cp.async.bulk.commit_group;" ::: "memory");
            // the shared memory must stay until the copies have read it; their writes to global memory
            // complete with the grid
            asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
        }
    }
    if (warp == 1) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols)
                                : "memory");
}

// 3-D map over q [num_tokens][num_heads][head_dim]: box = 64 columns x G heads x 128/G tokens,
// which lands as 128 rows (token-major, head-minor) of 128 bytes per 64-column chunk.
bool encode_q_map(CUtensorMap* map, const void* q, int head_dim, int num_heads, int num_tokens, int G) {
    EncodeTiledFn enc = encode_tiled_fn();
    if (!enc) return false;
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(head_dim), static_cast<cuuint64_t>(num_heads),
                                static_cast<cuuint64_t>(num_tokens)};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(head_dim) * 2,
                                   static_cast<cuuint64_t>(num_heads) * head_dim * 2};
    const cuuint32_t box[3] = {64, static_cast<cuuint32_t>(G), static_cast<cuuint32_t>(kRows / G)};
    const cuuint32_t estr[3] = {1, 1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT16, 3, const_cast<void*>(q), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 4-D map over a 16-bit pool [num_blocks][num_kv_heads][block_size][head_dim]: box = 64 columns x
// one block of one KV head; the block id is the outermost coordinate.
bool encode_pool_map16(CUtensorMap* map, const void* pool, int head_dim, int block_size, int num_kv_heads,
                       int num_blocks) {
    EncodeTiledFn enc = encode_tiled_fn();
    if (!enc) return false;
    const cuuint64_t dims[4] = {static_cast<cuuint64_t>(head_dim), static_cast<cuuint64_t>(block_size),
                                static_cast<cuuint64_t>(num_kv_heads), static_cast<cuuint64_t>(num_blocks)};
    const cuuint64_t strides[3] = {static_cast<cuuint64_t>(head_dim) * 2,
                                   static_cast<cuuint64_t>(block_size) * head_dim * 2,
                                   static_cast<cuuint64_t>(num_kv_heads) * block_size * head_dim * 2};
    const cuuint32_t box[4] = {64, static_cast<cuuint32_t>(block_size), 1, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT16, 4, const_cast<void*>(pool), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D, int BS, bool kBf16, bool kSplitP>
pkv_status launch_prefill(const PrefillArgs& a, const CUtensorMap& qm, const CUtensorMap& km, const CUtensorMap& vm,
                          const CUtensorMap& om, dim3 grid, cudaStream_t st) {
    auto kern = paged_prefill_kernel<D, BS, kBf16, kSplitP>;
    const uint32_t smem = PGeo<D>::kSmemBytes;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
        return PKV_ERR_CUDA;
    return launch_pdl(kern, grid, dim3(kPThreads), smem, st, a, qm, km, vm, om) == cudaSuccess ? PKV_OK
                                                                                             : PKV_ERR_CUDA;
}

template <int D, int BS>
pkv_status dispatch_mode(bool bf16, bool v_f16, const PrefillArgs& a, const CUtensorMap& qm, const CUtensorMap& km,
                         const CUtensorMap& vm, const CUtensorMap& om, dim3 grid, cudaStream_t st) {
    if (!bf16) return launch_prefill<D, BS, false, false>(a, qm, km, vm, om, grid, st);
    return v_f16 ? launch_prefill<D, BS, true, false>(a, qm, km, vm, om, grid, st)
                 : launch_prefill<D, BS, true, true>(a, qm, km, vm, om, grid, st);
}

// ---- narrowing a bf16 V to f16 (the workspace path of pkv_paged_attn_prefill) -------------

constexpr int kNarrowThreads = 256;
constexpr int kNarrowChunk = 16;       // table slots per CTA of the two passes
constexpr int kNarrowUnroll = 8;       // 16-byte loads each thread has in flight

// The chunk's block ids (slots j0 .. j0 + kNarrowChunk - 1) into shared memory, -1 for slots past
// the sequence's last reachable block (jn) and for ids outside the pool (reported when `err`).
__device__ __forceinline__ void load_chunk_ids(int* pids, const int32_t* __restrict__ trow, int j0, int jn,
                                               int num_blocks, uint32_t* err) {
    if (threadIdx.x < kNarrowChunk) {
        const int j = j0 + static_cast<int>(threadIdx.x);
        int pid = j < jn ? __ldg(trow + j) : -1;
        if (j < jn && (pid < 0 || pid >= num_blocks)) {
            if (err) raise_error(err, PKV_DEVERR_BLOCK_ID);
            pid = -1;
        }
        pids[threadIdx.x] = pid;
    }
    __syncthreads();
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

struct NarrowLayout {                  // the workspace of the bf16 path, in this order
    size_t pool, table, mult, parts, total;
    int chunks;
};

NarrowLayout narrow_layout(int num_seqs, int maxb, int num_kv_heads, int head_dim, int block_size) {
    NarrowLayout l{};
    const size_t blocks = static_cast<size_t>(num_seqs) * maxb;
    const size_t sh = static_cast<size_t>(num_seqs) * num_kv_heads;
    l.chunks = (maxb + kNarrowChunk - 1) / kNarrowChunk;
    l.pool = align256(blocks * num_kv_heads * block_size * head_dim * 2);
    l.table = align256(blocks * sizeof(int32_t));
    l.mult = align256(sh * sizeof(float));
    l.parts = align256(sh * l.chunks * sizeof(uint32_t));
    l.total = l.pool + l.table + l.mult + l.parts;
    return l;
}

// The largest finite magnitude among 8 bf16 values (as the bits of |v|; bf16 magnitudes order as
// integers); 0 for a unit that does not count (its key position is past the context, or its block
// id is bad).
__device__ __forceinline__ uint32_t absmax8(const uint4& x, bool valid) {
    if (!valid) return 0;
    const uint32_t w[4] = {x.x, x.y, x.z, x.w};
    uint32_t m = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint32_t lo = w[i] & 0x7fffu, hi = (w[i] >> 16) & 0x7fffu;
        m = max(m, lo < 0x7f80u ? lo : 0u);   // exponent all ones: Inf or NaN, not scaled for
        m = max(m, hi < 0x7f80u ? hi : 0u);
    }
    return m;
}

// Pass 1: for each (sequence s, KV head h, chunk of kNarrowChunk table slots) the largest finite
// |v| of the V rows at positions < L_s, into parts[(s, h)][chunk].
template <int BS, int D>
__global__ void __launch_bounds__(kNarrowThreads)
v_absmax_kernel(const uint4* __restrict__ v_pool, const int32_t* __restrict__ tables,
                const int32_t* __restrict__ lens, uint32_t* __restrict__ parts, int maxb, int num_kv_heads,
                int num_blocks) {
    constexpr int kRun = BS * D / 8;                 // 16-byte units of one block and head
    pdl_trigger();
    pdl_wait();                                      // the pool may still be written by the previous kernel
    const int chunk = blockIdx.x, h = blockIdx.y, s = blockIdx.z;
    const int L = __ldg(lens + s);
    const long long cap = static_cast<long long>(maxb) * BS;
    const int nb = L <= 0 ? 0 : static_cast<int>((min(static_cast<long long>(L), cap) + BS - 1) / BS);
    const int j0 = chunk * kNarrowChunk, j1 = min(nb, j0 + kNarrowChunk);
    __shared__ int pids[kNarrowChunk];
    load_chunk_ids(pids, tables + static_cast<size_t>(s) * maxb, j0, j1, num_blocks, nullptr);
    uint32_t m = 0;
    for (int u0 = threadIdx.x; u0 < (j1 - j0) * kRun; u0 += kNarrowThreads * kNarrowUnroll) {
        uint4 x[kNarrowUnroll];
        bool valid[kNarrowUnroll];
#pragma unroll
        for (int k = 0; k < kNarrowUnroll; ++k) {
            const int u = u0 + k * kNarrowThreads;
            const int jj = u / kRun, e = u % kRun;
            valid[k] = false;
            if (u < (j1 - j0) * kRun) {
                const int pid = pids[jj];
                valid[k] = pid >= 0 && (j0 + jj) * BS + e / (D / 8) < L;
                if (valid[k])
                    x[k] = __ldg(v_pool + ((static_cast<size_t>(pid) * num_kv_heads + h) * kRun + e));
            }
        }
#pragma unroll
        for (int k = 0; k < kNarrowUnroll; ++k) m = max(m, absmax8(x[k], valid[k]));
    }
    m = __reduce_max_sync(0xffffffffu, m);
    __shared__ uint32_t wm[kNarrowThreads / 32];
    if ((threadIdx.x & 31) == 0) wm[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int w = 1; w < kNarrowThreads / 32; ++w) m = max(m, wm[w]);
        parts[(static_cast<size_t>(s) * num_kv_heads + h) * gridDim.x + chunk] = m;
    }
}

// The power of two e with which v * 2^-e fits f16: the largest finite |v| (bf16 bits) lands in
// [2^15, 2^16), so no value overflows and every value down to 2^-29 of the largest stays a normal
// f16 (exact: bf16 carries 8 significant bits, f16 11).  Clamped so that 2^e and 2^-e are normal
// floats; 0 for a head without finite values.
__device__ __forceinline__ int narrow_exponent(uint32_t maxbits) {
    if (maxbits == 0) return 0;
    const int eb = static_cast<int>(maxbits >> 7);   // biased bf16 exponent, 0 for subnormals
    const int e = (eb == 0 ? -126 : eb - 127) - 15;
    return min(max(e, -96), 112);
}

// Pass 2: the same slots; V rows at positions < L_s become f16(v * 2^-e) in the workspace pool
// (block s * maxb + j), later rows zeros; the workspace table and the output factor 2^e are
// written alongside.  A bad block id leaves a -1 in the workspace table, which the prefill kernel
// reports; raised here too.
template <int BS, int D>
__global__ void __launch_bounds__(kNarrowThreads)
v_narrow_kernel(const uint4* __restrict__ v_pool, const int32_t* __restrict__ tables,
                const int32_t* __restrict__ lens, const uint32_t* __restrict__ parts, uint4* __restrict__ wv,
                int32_t* __restrict__ wtab, float* __restrict__ mult, int maxb, int num_kv_heads, int num_blocks,
                uint32_t* err) {
    constexpr int kRun = BS * D / 8;
    pdl_trigger();
    pdl_wait();                                      // every partial maximum is written
    const int chunk = blockIdx.x, h = blockIdx.y, s = blockIdx.z;
    const size_t sh = static_cast<size_t>(s) * num_kv_heads + h;
    __shared__ float down;
    if (threadIdx.x < 32) {
        uint32_t m = 0;
        for (int c = threadIdx.x; c < static_cast<int>(gridDim.x); c += 32) m = max(m, __ldg(parts + sh * gridDim.x + c));
        m = __reduce_max_sync(0xffffffffu, m);
        if (threadIdx.x == 0) {
            const int e = narrow_exponent(m);
            down = __uint_as_float(static_cast<uint32_t>(127 - e) << 23);    // 2^-e
            if (chunk == 0) mult[sh] = __uint_as_float(static_cast<uint32_t>(127 + e) << 23);   // 2^e
        }
    }
    __syncthreads();
    const float f = down;
    const int L = __ldg(lens + s);
    const long long cap = static_cast<long long>(maxb) * BS;
    const int nb = L <= 0 ? 0 : static_cast<int>((min(static_cast<long long>(L), cap) + BS - 1) / BS);
    const int j0 = chunk * kNarrowChunk, j1 = min(maxb, j0 + kNarrowChunk);
    const int jn = min(nb, j1);
    __shared__ int pids[kNarrowChunk];
    load_chunk_ids(pids, tables + static_cast<size_t>(s) * maxb, j0, jn, num_blocks, h == 0 ? err : nullptr);
    if (h == 0 && static_cast<int>(threadIdx.x) < j1 - j0)
        wtab[static_cast<size_t>(s) * maxb + j0 + threadIdx.x] =
            pids[threadIdx.x] >= 0 ? static_cast<int32_t>(s * maxb + j0 + threadIdx.x) : -1;
    for (int u0 = threadIdx.x; u0 < (jn - j0) * kRun; u0 += kNarrowThreads * kNarrowUnroll) {
        uint4 x[kNarrowUnroll];
        int dst[kNarrowUnroll];                      // -1: nothing to write; else the unit's index in the chunk
        bool live[kNarrowUnroll];
#pragma unroll
        for (int k = 0; k < kNarrowUnroll; ++k) {
            const int u = u0 + k * kNarrowThreads;
            dst[k] = -1;
            live[k] = false;
            if (u < (jn - j0) * kRun) {
                const int jj = u / kRun, e = u % kRun;
                const int pid = pids[jj];
                if (pid >= 0) {
                    dst[k] = u;
                    live[k] = (j0 + jj) * BS + e / (D / 8) < L;
                    if (live[k]) x[k] = __ldg(v_pool + ((static_cast<size_t>(pid) * num_kv_heads + h) * kRun + e));
                }
            }
        }
#pragma unroll
        for (int k = 0; k < kNarrowUnroll; ++k) {
            if (dst[k] < 0) continue;
            const int j = j0 + dst[k] / kRun, e = dst[k] % kRun;
            uint4 o = make_uint4(0u, 0u, 0u, 0u);
            if (live[k]) {
                const uint32_t w[4] = {x[k].x, x[k].y, x[k].z, x[k].w};
                uint32_t r[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const __half2 v = __floats2half2_rn(__uint_as_float(w[i] << 16) * f,
                                                        __uint_as_float(w[i] & 0xffff0000u) * f);
                    r[i] = *reinterpret_cast<const uint32_t*>(&v);
                }
                o = make_uint4(r[0], r[1], r[2], r[3]);
            }
            wv[((static_cast<size_t>(s) * maxb + j) * num_kv_heads + h) * kRun + e] = o;
        }
    }
}

template <int BS, int D>
pkv_status launch_narrow(const void* v_pool, const int32_t* tables, const int32_t* lens, uint8_t* ws,
                         const NarrowLayout& l, int num_seqs, int maxb, int num_kv_heads, int num_blocks,
                         uint32_t* err, cudaStream_t st) {
    const dim3 grid(static_cast<unsigned>(l.chunks), static_cast<unsigned>(num_kv_heads),
                    static_cast<unsigned>(num_seqs));
    uint4* wv = reinterpret_cast<uint4*>(ws);
    int32_t* wtab = reinterpret_cast<int32_t*>(ws + l.pool);
    float* mult = reinterpret_cast<float*>(ws + l.pool + l.table);
    uint32_t* parts = reinterpret_cast<uint32_t*>(ws + l.pool + l.table + l.mult);
    if (launch_pdl(v_absmax_kernel<BS, D>, grid, dim3(kNarrowThreads), 0, st, static_cast<const uint4*>(v_pool),
                   tables, lens, parts, maxb, num_kv_heads, num_blocks) != cudaSuccess)
        return PKV_ERR_CUDA;
    return launch_pdl(v_narrow_kernel<BS, D>, grid, dim3(kNarrowThreads), 0, st, static_cast<const uint4*>(v_pool),
                      tables, lens, static_cast<const uint32_t*>(parts), wv, wtab, mult, maxb, num_kv_heads,
                      num_blocks, err) == cudaSuccess
               ? PKV_OK
               : PKV_ERR_CUDA;
}

}  // namespace

pkv_status prefill_check(const PrefillLaunch& p, bool dtype_supported) {
    if (p.num_seqs < 0 || p.num_tokens < 0 || p.max_query_len < 0 || p.num_heads <= 0 || p.num_kv_heads <= 0 ||
        p.num_blocks <= 0 || p.max_blocks_per_seq <= 0 || !(p.scale > 0.f) || !std::isfinite(p.scale))
        return PKV_ERR_INVALID_ARG;
    if (p.num_heads % p.num_kv_heads != 0) return PKV_ERR_INVALID_ARG;
    if (!dtype_supported) return PKV_ERR_UNSUPPORTED;
    const int G = p.num_heads / p.num_kv_heads;
    if ((p.head_dim != 64 && p.head_dim != 128) || (p.block_size != 16 && p.block_size != 32) ||
        (G != 1 && G != 2 && G != 4 && G != 8 && G != 16))
        return PKV_ERR_UNSUPPORTED;
    if (p.num_seqs == 0 || p.num_tokens == 0 || p.max_query_len == 0) return PKV_OK;
    if (!p.out || !p.q || !p.k_pool || !p.v_pool || !p.k_tables || !p.context_lens || !p.query_start)
        return PKV_ERR_INVALID_ARG;
    if (!aligned16(p.out) || !aligned16(p.q) || !aligned16(p.k_pool) || !aligned16(p.v_pool) ||
        (reinterpret_cast<uintptr_t>(p.k_tables) & 3) || (reinterpret_cast<uintptr_t>(p.context_lens) & 3) ||
        (reinterpret_cast<uintptr_t>(p.query_start) & 3) || (reinterpret_cast<uintptr_t>(p.err) & 3))
        return PKV_ERR_ALIGNMENT;
    const long long tiles = (static_cast<long long>(p.max_query_len) * G + kTiles * kRows - 1) / (kTiles * kRows);
    if (p.num_seqs > 65535 || p.num_kv_heads > 65535 || tiles > 0x7fffffffLL ||
        static_cast<long long>(p.num_seqs) * p.max_blocks_per_seq > 0x7fffffffLL)
        return PKV_ERR_INVALID_ARG;
    return PKV_OK;
}

pkv_status prefill_launch(const PrefillLaunch& p) {
    const int G = p.num_heads / p.num_kv_heads;
    const long long tiles = (static_cast<long long>(p.max_query_len) * G + kTiles * kRows - 1) / (kTiles * kRows);
    PrefillArgs a{};
    a.out = p.out;
    a.block_tables = p.k_tables;
    a.v_tables = p.v_tables ? p.v_tables : p.k_tables;
    a.context_lens = p.context_lens;
    a.query_start = p.query_start;
    a.v_mult = p.v_mult;
    a.err = p.err;
    a.max_blocks_per_seq = p.max_blocks_per_seq;
    a.num_tokens = p.num_tokens;
    a.num_heads = p.num_heads;
    a.num_blocks = p.num_blocks;
    a.v_num_blocks = p.v_tables ? p.v_num_blocks : p.num_blocks;
    a.group = G;
    a.scale_log2 = p.scale * 1.4426950408889634f;
    a.v_mult_all = p.v_mult_all;

    alignas(64) CUtensorMap qm;
    alignas(64) CUtensorMap km;
    alignas(64) CUtensorMap vm;
    alignas(64) CUtensorMap om;   // the output has q's layout, so it is stored with q's box
    if (!encode_q_map(&qm, p.q, p.head_dim, p.num_heads, p.num_tokens, G) ||
        !encode_pool_map16(&km, p.k_pool, p.head_dim, p.block_size, p.num_kv_heads, p.num_blocks) ||
        !encode_pool_map16(&vm, p.v_pool, p.head_dim, p.block_size, p.num_kv_heads, a.v_num_blocks) ||
        !encode_q_map(&om, p.out, p.head_dim, p.num_heads, p.num_tokens, G))
        return PKV_ERR_CUDA;
    const dim3 grid(static_cast<unsigned>(tiles), static_cast<unsigned>(p.num_kv_heads),
                    static_cast<unsigned>(p.num_seqs));
    cudaStream_t st = p.stream;
    if (p.head_dim == 128)
        return p.block_size == 16 ? dispatch_mode<128, 16>(p.bf16, p.v_f16, a, qm, km, vm, om, grid, st)
                                  : dispatch_mode<128, 32>(p.bf16, p.v_f16, a, qm, km, vm, om, grid, st);
    return p.block_size == 16 ? dispatch_mode<64, 16>(p.bf16, p.v_f16, a, qm, km, vm, om, grid, st)
                              : dispatch_mode<64, 32>(p.bf16, p.v_f16, a, qm, km, vm, om, grid, st);
}

}  // namespace pkv

extern "C" size_t pkv_prefill_workspace_bytes(pkv_dtype dtype, int num_seqs, int max_blocks_per_seq,
                                              int num_kv_heads, int head_dim, int block_size) {
    if (dtype != PKV_BF16 || num_seqs <= 0 || max_blocks_per_seq <= 0 || num_kv_heads <= 0 || head_dim <= 0 ||
        block_size <= 0)
        return 0;
    return pkv::narrow_layout(num_seqs, max_blocks_per_seq, num_kv_heads, head_dim, block_size).total;
}

extern "C" pkv_status pkv_paged_attn_prefill(void* out, const void* q, pkv_dtype dtype, const void* k_pool,
                                             const void* v_pool, const int32_t* block_tables, int max_blocks_per_seq,
                                             const int32_t* context_lens, const int32_t* query_start,
                                             int max_query_len, int num_seqs, int num_tokens, int num_heads,
                                             int num_kv_heads, int head_dim, int block_size, int num_blocks,
                                             float scale, void* workspace, size_t workspace_bytes,
                                             uint32_t* device_error, void* stream) {
    using namespace pkv;
    PrefillLaunch p{};
    p.out = out;
    p.q = q;
    p.bf16 = dtype == PKV_BF16;
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
    p.scale = scale;
    p.v_mult_all = 1.f;
    p.err = device_error;
    p.stream = static_cast<cudaStream_t>(stream);
    p.v_f16 = !p.bf16;
    const pkv_status chk = prefill_check(p, dtype == PKV_F16 || dtype == PKV_BF16);
    if (chk != PKV_OK || num_seqs == 0 || num_tokens == 0 || max_query_len == 0) return chk;
    if (p.bf16 && workspace) {
        // V narrowed to f16 with a power-of-two scale per (sequence, KV head): one f16 P.V product
        const NarrowLayout l = narrow_layout(num_seqs, max_blocks_per_seq, num_kv_heads, head_dim, block_size);
        if (workspace_bytes < l.total) return PKV_ERR_WORKSPACE;
        if (reinterpret_cast<uintptr_t>(workspace) & 255) return PKV_ERR_ALIGNMENT;
        uint8_t* ws = static_cast<uint8_t*>(workspace);
        pkv_status st;
        if (head_dim == 128)
            st = block_size == 16 ? launch_narrow<16, 128>(v_pool, block_tables, context_lens, ws, l, num_seqs,
                                                           max_blocks_per_seq, num_kv_heads, num_blocks,
                                                           device_error, p.stream)
                                  : launch_narrow<32, 128>(v_pool, block_tables, context_lens, ws, l, num_seqs,
                                                           max_blocks_per_seq, num_kv_heads, num_blocks,
                                                           device_error, p.stream);
        else
            st = block_size == 16 ? launch_narrow<16, 64>(v_pool, block_tables, context_lens, ws, l, num_seqs,
                                                          max_blocks_per_seq, num_kv_heads, num_blocks, device_error,
                                                          p.stream)
                                  : launch_narrow<32, 64>(v_pool, block_tables, context_lens, ws, l, num_seqs,
                                                          max_blocks_per_seq, num_kv_heads, num_blocks, device_error,
                                                          p.stream);
        if (st != PKV_OK) return st;
        p.v_pool = ws;
        p.v_tables = reinterpret_cast<const int32_t*>(ws + l.pool);
        p.v_num_blocks = num_seqs * max_blocks_per_seq;
        p.v_mult = reinterpret_cast<const float*>(ws + l.pool + l.table);
        p.v_f16 = true;
    }
    return prefill_launch(p);
}
