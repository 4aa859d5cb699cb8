// pkv_paged_attn_decode: single-query attention over the paged KV pool.
//
// What it computes is the token form of causal attention for the last token
// of each sequence (Wikipedia "PagedAttention", section "Mathematical
// formulation"): o = sum_t softmax_t(scale q.k_t) v_t over the L cached tokens,
// read block by block through the block table.  The page's block form (A_ij
// over ceil(i/B) blocks) is the same sum grouped by block; this kernel groups
// it further by partition and merges partitions exactly with log-sum-exp.
//
// Design (sm_100a):
//   * Work unit = (partition of <= partition_size tokens, KV head, sequence).
//     All G query heads of the KV head ride in the same CTA, so each K/V tile
//     crosses HBM once per group (GQA; glossary "PagedAttention", section
//     "Related methods").  A CTA streams one partition, or, when the caller
//     states partitions smaller than the automatic size, as many consecutive
//     ones as that size holds: the ring keeps streaming across them and each
//     still ends in its own partial, merged exactly afterwards.  CTAs are
//     dispatched partition index last-first.
//   * One producer warp issues TMA tile loads.  The pool is described to TMA
//     as a 4-D tensor [head_dim, block_size, num_kv_heads, num_blocks]; the
//     block-table indirection is simply the outermost tile coordinate.  Tiles
//     land in shared memory with 128-byte swizzling, in a ring of stages
//     guarded by transaction barriers (full: TMA bytes arrived; empty:
//     consumer done), with evict-first L2 hints since the KV is streamed once.
//   * Four consumer warps take ring stages round-robin (a stage is one block,
//     or two when a block's K+V tiles are under 8 KB).  Each computes
//     S^T = K Q^T with mma.sync m16n8k16 (16 tokens as M, the query heads of
//     the group as N in tiles of 8, head_dim as K), an online softmax in
//     registers per head (running max and sum, base-2 exponent, output
//     rescaled only when a running max moved), and O^T += V^T P^T with the P^T
//     fragments made from the S^T accumulators by movmatrix transposes.
//   * 16-bit tiles are read with ldmatrix (K) and ldmatrix.trans (V^T) from
//     the swizzled tile; every 8-lane phase touches 8 distinct bank groups.
//     FP8 E4M3 tiles are read with 16-byte shared loads and widened to f16
//     (or bf16) in registers, two values per instruction, so the MMA sees
//     exact values and no dequantised copy is written anywhere; for them the
//     head_dim axis of QK and of the output is permuted (the same permutation
//     on both operands, undone on output) so that each lane's fragment comes
//     from contiguous bytes.
//   * At the end of each partition the four warps' states are merged in a
//     shared-memory buffer of their own (a named barrier among the consumer
//     warps; the producer keeps filling the ring); a CTA that covers its whole
//     sequence writes the output, otherwise it writes (max, sum, normalised
//     output) to the workspace and a second small kernel merges the
//     partitions.
//   * Masking: slots past the context length in the last block get score
//     -inf (by select) and their V rows are zeroed before the MMA, so
//     arbitrary bit patterns in unused slots (NaN/Inf) cannot leak.
//   * Every barrier wait is bounded; a bad table entry or context length is
//     reported through the device error word and yields NaN output for that
//     (sequence, head group), never a trap or an out-of-bounds read.

#include <cuda_runtime.h>

#include <cmath>
#include <mutex>

#include "pkv_device.cuh"
#include "pkv_host.h"

namespace pkv {
namespace {

// 2^x on the exponential unit (PTX ex2.approx.ftz: results below 2^-126 flush to zero)
__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Occupancy plan: the kernel streams HBM through TMA, so what keeps the memory
// system busy is the number of consumer warps ready to drain the ring.  With
// query groups of up to 8 heads a CTA fits in 96 registers per thread and a
// 32 KB ring, so four CTAs share an SM; larger groups hold twice the
// accumulators and run two CTAs with 64 KB rings.  PKV_RING_BYTES and
// PKV_MIN_CTAS override the plan for every instance (used for tuning sweeps).

constexpr int kConsumerWarps = 4;
constexpr int kThreads = (kConsumerWarps + 1) * 32;

enum KvKind { KV_F16 = 0, KV_BF16 = 1, KV_E4M3 = 2 };

struct DecodeArgs {
    void* out;
    const void* q;
    const int32_t* block_tables;
    const int32_t* context_lens;
    float* ws_o;      // [S][H][max_partitions][D]
    float2* ws_ml;    // [S][H][max_partitions] (max in log2 units, sum)
    uint32_t* err;
    int max_blocks_per_seq, max_context_len, num_seqs, num_heads, num_kv_heads, num_blocks;
    int block_size, partition_size, max_partitions;
    float qk_scale_log2;  // scale * k_scale * log2(e)
    float v_scale;        // 1 for 16-bit pools
    // shared-prefix decode (all null / zero in the plain call)
    const int32_t* seq_start;   // [S] first token each sequence attends in this pass (its shared prefix length)
    const int32_t* unit_seqs;   // prefix pass: [units][unit_width] member sequences of each unit, -1 pads
    const int32_t* unit_len;    // prefix pass: [units] shared tokens of each unit
    int unit_width;
    int slot_base;              // first partition slot of the workspace this pass writes
    int prefix_partition_size;  // tail pass and merge: partition size of the prefix pass
    int max_prefix_len;         // bound of every unit_len and seq_start (0 in the plain call)
    int parts_per_cta;          // consecutive partitions one CTA streams (each still gets its own partial)
};

// Written by the tail pass into every prefix slot a sequence's merge will read, before the
// prefix pass runs: a slot still holding it was not covered by a unit (max NaN, sum -1).
constexpr uint32_t kUnwrittenSum = 0xbf800000u;   // -1.0f

// ---- MMA and conversions ------------------------------------------------------

template <bool kBf16>
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    if constexpr (kBf16)
        asm volatile(
            "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
            "{%0,%1,%2,%3};"
            : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
            : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
    else
        asm volatile(
            "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
            "{%0,%1,%2,%3};"
            : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
            : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Four E4M3 values (bytes of x, low byte first) -> two MMA operand words: lo holds
// bytes 0-1, hi bytes 2-3, each as a pair of 16-bit values (exact widening).
template <bool kBf16>
__device__ __forceinline__ void widen_e4m3x4(uint32_t x, uint32_t& lo, uint32_t& hi) {
    uint32_t h0, h1;
    asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %2;\n\t"
        "cvt.rn.f16x2.e4m3x2 %0, l;\n\tcvt.rn.f16x2.e4m3x2 %1, h;\n\t}"
        : "=r"(h0), "=r"(h1)
        : "r"(x));
    if constexpr (!kBf16) {
        lo = h0;
        hi = h1;
    } else {
        const float2 f0 = __half22float2(*reinterpret_cast<const __half2*>(&h0));
        const float2 f1 = __half22float2(*reinterpret_cast<const __half2*>(&h1));
        const __nv_bfloat162 b0 = __floats2bfloat162_rn(f0.x, f0.y);
        const __nv_bfloat162 b1 = __floats2bfloat162_rn(f1.x, f1.y);
        lo = *reinterpret_cast<const uint32_t*>(&b0);
        hi = *reinterpret_cast<const uint32_t*>(&b1);
    }
}

template <bool kBf16>
__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
    if constexpr (kBf16) {
        const __nv_bfloat162 b = __floats2bfloat162_rn(lo, hi);
        return *reinterpret_cast<const uint32_t*>(&b);
    } else {
        const __half2 h = __floats2half2_rn(lo, hi);
        return *reinterpret_cast<const uint32_t*>(&h);
    }
}

// bf16 keeps 8 significant bits: P = hi + lo with both parts bf16 keeps ~16.
__device__ __forceinline__ float bf16_residual(float x) {
    return x - __bfloat162float(__float2bfloat16_rn(x));
}

template <bool kBf16>
__device__ __forceinline__ void store_out(void* out, size_t idx, float v) {
    if constexpr (kBf16)
        static_cast<__nv_bfloat16*>(out)[idx] = __float2bfloat16_rn(v);
    else
        static_cast<__half*>(out)[idx] = __float2half_rn(v);
}

__device__ __forceinline__ uint32_t word(const uint4& v, int i) {
    return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w;
}

// ---- tile geometry ---------------------------------------------------------------

template <int KV, int D, int BS, bool kHi>
struct Geo {
    static constexpr int E = KV == KV_E4M3 ? 1 : 2;   // element bytes
    static constexpr int kNsub = D * E / 128;          // 128-byte sub-rows per token row
    static constexpr int kSubBytes = BS * 128;         // one swizzled sub-tile (BS rows x 128 B)
    static constexpr int kTileBytes = kNsub * kSubBytes;   // one (block, KV head) K or V tile
    // blocks per ring stage: small tiles are paired so a stage moves at least 8 KB
    static constexpr int kBps = 2 * kTileBytes >= 8192 ? 1 : 8192 / (2 * kTileBytes);
    static constexpr int kStageTok = kBps * BS;        // tokens per stage
    static constexpr int kStageBytes = 2 * kBps * kTileBytes;  // K tiles, then V tiles
    static constexpr int kKsteps = D / 16;             // k-steps of the QK contraction
    static constexpr int kMtTok = kStageTok / 16;      // 16-token m-tiles per stage (QK M, PV K)
    static constexpr int kMtDim = D / 16;              // 16-dim m-tiles of the output (PV M)
#ifdef PKV_RING_BYTES
    static constexpr int kRingTarget = PKV_RING_BYTES;
#else
    static constexpr int kRingTarget = kHi ? 65536 : 32768;
#endif
    static constexpr int kStagesRaw = kRingTarget / kStageBytes / kConsumerWarps * kConsumerWarps;
    static constexpr int kStages = kStagesRaw < 4 ? 4 : (kStagesRaw > 32 ? 32 : kStagesRaw);
    static constexpr int kRingBytes = kStages * kStageBytes;
    static constexpr int kRowsMax = kHi ? 16 : 8;                 // query rows of the instance
    // the consumers' partition merge has a buffer of its own: the producer keeps filling the ring
    // with the next partition's tiles meanwhile
    static constexpr int kMergeBytes = kConsumerWarps * kRowsMax * (D + 2) * 4;
    static constexpr int kDataBytes = kRingBytes + kMergeBytes;
    static constexpr int kSmemBytes = 1024 /* alignment slack */ + kDataBytes + kStages * 16 + 16;
    // CTAs per SM that the register budget must allow (shared memory permitting)
    static constexpr int kSmemCtas = (227 * 1024) / (kSmemBytes + 1024);
#ifdef PKV_MIN_CTAS
    static constexpr int kMinCtas = PKV_MIN_CTAS;
#else
    static constexpr int kMinCtas = (kHi ? 2 : 4) < kSmemCtas ? (kHi ? 2 : 4) : kSmemCtas;
#endif
    static_assert(D * E == 128 || D * E == 256, "row must be 128 or 256 bytes");
    static_assert(kStages % kConsumerWarps == 0, "stage -> warp mapping must be fixed");
    static_assert(kStageTok % 16 == 0, "a stage holds whole 16-token m-tiles");

    // Byte offset, inside a stage, of 16-byte chunk q of token t's K row (V: add kVOff).
    static constexpr int kVOff = kBps * kTileBytes;
    __device__ static __forceinline__ uint32_t at(int t, int q) {
        return static_cast<uint32_t>((t / BS) * kTileBytes + (q >> 3) * kSubBytes) + swz128(t % BS, q & 7);
    }
    // QK contraction: head_dim index of b0's first element for quad lane c at k-step ks
    // (b1 starts kQkB1 elements later).  16-bit tiles use the natural order (fragments
    // come from ldmatrix); FP8 tiles use a permuted order in which each lane's four
    // k-values of a k-step are four consecutive bytes of the row.
    __device__ static __forceinline__ int qk_dim(int c, int ks) { return E == 2 ? ks * 16 + 2 * c : 32 * c + 4 * ks; }
    static constexpr int kQkB1 = E == 2 ? 8 : 2;
    // PV output: head_dim index held in row rr (0..15) of output m-tile md.
    __device__ static __forceinline__ int o_dim(int md, int rr) {
        return E == 2 ? md * 16 + rr : 16 * (rr & 7) + 2 * md + (rr >> 3);
    }
};

__device__ __forceinline__ void ldsm_x4(uint32_t (&a)[4], uint32_t addr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(a[0]), "=r"(a[1]), "=r"(a[2]), "=r"(a[3])
                 : "r"(addr)
                 : "memory");
}

__device__ __forceinline__ void ldsm_x4_trans(uint32_t (&a)[4], uint32_t addr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(a[0]), "=r"(a[1]), "=r"(a[2]), "=r"(a[3])
                 : "r"(addr)
                 : "memory");
}

// Transpose of an 8x8 16-bit matrix held one row pair per lane (lane/4 = row).
__device__ __forceinline__ uint32_t movmatrix_t(uint32_t x) {
    uint32_t y;
    asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
    return y;
}

// Zero the 16-bit halves whose token is masked: lo half = token t, hi half = token t + 1.
__device__ __forceinline__ uint32_t mask_pair(uint32_t x, int t, int valid) {
    const uint32_t lo = t < valid ? 0x0000ffffu : 0u;
    const uint32_t hi = t + 1 < valid ? 0xffff0000u : 0u;
    return x & (lo | hi);
}

// Named barrier of the four consumer warps (the producer warp keeps streaming meanwhile).
__device__ __forceinline__ void consumer_barrier() {
    asm volatile("bar.sync 1, %0;" ::"n"(kConsumerWarps * 32) : "memory");
}

// ---- pass 1: one CTA per (partition, KV head, sequence) ------------------------------

template <int KV, bool kQBf16, int D, int BS, bool kHi>
__global__ void __launch_bounds__(kThreads, (Geo<KV, D, BS, kHi>::kMinCtas))
paged_decode_kernel(const DecodeArgs a, const __grid_constant__ CUtensorMap kmap,
                    const __grid_constant__ CUtensorMap vmap) {
    using Gm = Geo<KV, D, BS, kHi>;
    constexpr bool kBf16 = (KV == KV_BF16) || (KV == KV_E4M3 && kQBf16);
    constexpr int NST = Gm::kStages;
    constexpr int NTH = kHi ? 2 : 1;   // 8-head n-tiles of the query group

    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_addr(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* gbase = smem_raw + (base - raw);
    const uint32_t bar_full = base + Gm::kDataBytes;
    const uint32_t bar_empty = bar_full + NST * 8;
    volatile int* s_abort = reinterpret_cast<volatile int*>(gbase + Gm::kDataBytes + NST * 16);

    // grid (KV heads, sequences or units, partition groups): the partition index is dispatched last
    // first, so short trailing work does not end the grid behind long CTAs
    const int part = static_cast<int>(gridDim.z - 1 - blockIdx.z), kvh = blockIdx.x, z = blockIdx.y;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = a.num_heads / a.num_kv_heads;
    const int H = a.num_heads;
    // The CTA's query rows: the G heads of sequence z, or (prefix pass) the G heads of
    // every member of prefix unit z.  Tokens [start, start + L) of table row `tseq`.
    const bool prefix_pass = a.unit_seqs != nullptr;
    int rows = G, L, start = 0, tseq = z;
    bool bad_len;
    // A grid must not complete before the kernel ahead of it on the stream has (the merge, and
    // the next call, rely on that ordering through both passes): CTAs with work pass pdl_wait(),
    // and of the CTAs that leave early, CTA (0, 0, 0) waits too, so at least one CTA of every
    // grid does; the others leave at once and free their slots.
    const bool first_cta = blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0;
    if (prefix_pass) {
        // members: valid sequence ids packed first, -1 pads after them; each member's own prefix
        // length must be the unit's (seq_start holds seq_prefix_len here)
        const int32_t* mem = a.unit_seqs + static_cast<size_t>(z) * a.unit_width;
        tseq = __ldg(mem);
        L = __ldg(a.unit_len + z);
        int members = 0;
        bool bad_member = false, padded = false;
        for (int m = 0; m < a.unit_width; ++m) {
            const int id = __ldg(mem + m);
            if (id < 0) {
                padded = true;
                continue;
            }
            ++members;
            bad_member |= padded || id >= a.num_seqs || (a.seq_start && __ldg(a.seq_start + id) != L);
        }
        rows = members * G;
        bad_len = members == 0 || bad_member || L < 0 || L % BS != 0 || L > a.max_blocks_per_seq * BS ||
                  L > a.max_prefix_len;
        if (bad_len || L == 0 || grid_timed_out(a.err)) {
            if (bad_len && part == 0 && threadIdx.x == 0) raise_error(a.err, PKV_DEVERR_CONTEXT_LEN);
            if (first_cta) pdl_wait();
            return;   // the members' prefix slots keep the tail pass's marker: their merges give NaN
        }
    } else {
        const int Lt = __ldg(a.context_lens + z);
        start = a.seq_start ? __ldg(a.seq_start + z) : 0;
        bad_len = Lt < 0 || Lt > a.max_blocks_per_seq * BS || Lt > a.max_context_len || start < 0 || start > Lt ||
                  start % BS != 0 || start > a.max_prefix_len;
        L = Lt - start;
        if (!bad_len && start > 0 && part == 0) {
            // mark the prefix slots this sequence's merge reads; the prefix pass (next on the
            // stream) overwrites those of the units that cover it
            pdl_wait();
            const int np_pre = (start + a.prefix_partition_size - 1) / a.prefix_partition_size;
            const size_t row0 = static_cast<size_t>(z) * H + static_cast<size_t>(kvh) * G;
            for (int e = threadIdx.x; e < G * np_pre; e += kThreads)
                a.ws_ml[(row0 + e / np_pre) * a.max_partitions + e % np_pre] =
                    make_float2(__int_as_float(0x7fc00000), __uint_as_float(kUnwrittenSum));
        }
        const bool give_up = grid_timed_out(a.err);
        if (bad_len || L == 0 || give_up) {
            if (part == 0 && (start == 0 || bad_len)) {
                pdl_wait();
                if (bad_len && threadIdx.x == 0) raise_error(a.err, PKV_DEVERR_CONTEXT_LEN);
                const float v = (bad_len || give_up) ? __int_as_float(0x7fc00000) : 0.f;
                const size_t row0 = static_cast<size_t>(z) * H + static_cast<size_t>(kvh) * G;
                for (int e = threadIdx.x; e < G * D; e += kThreads) store_out<kQBf16>(a.out, row0 * D + e, v);
            } else if (first_cta) {
                pdl_wait();
            }
            return;
        }
    }
    // global q / out row of CTA row r
    auto row_of = [&](int r) -> size_t {
        if (!prefix_pass) return static_cast<size_t>(z) * H + static_cast<size_t>(kvh) * G + r;
        const int m = r / G;
        return static_cast<size_t>(__ldg(a.unit_seqs + static_cast<size_t>(z) * a.unit_width + m)) * H +
               static_cast<size_t>(kvh) * G + (r - m * G);
    };
    // the CTA streams partitions part0 .. part0 + nlp - 1 (consecutive, one partial each)
    const int PS = a.partition_size;
    const int nparts = (L + PS - 1) / PS;
    const int part0 = part * a.parts_per_cta;
    if (part0 >= nparts) {
        if (first_cta) pdl_wait();
        return;
    }
    const int nlp = min(a.parts_per_cta, nparts - part0);
    const int tok_begin = part0 * PS;
    const int tok_end = min(L, tok_begin + nlp * PS);
    const int nblk = (tok_end - tok_begin + BS - 1) / BS;
    const int nstage = (nblk + Gm::kBps - 1) / Gm::kBps;
    const int blk0 = (start + tok_begin) / BS;

    if (threadIdx.x == 0) {
#pragma unroll
        for (int i = 0; i < NST; ++i) {
            mbar_init(bar_full + 8 * i, 1);
            mbar_init(bar_empty + 8 * i, 1);
        }
        *s_abort = 0;
        mbar_fence_init();
    }
    __syncthreads();

    // Per-warp softmax state.  Lane (r = lane/4, c = lane%4) owns query heads
    // nh*8 + 2c and nh*8 + 2c + 1 and, in the output, head_dim rows o_dim(md, r) and
    // o_dim(md, r + 8) of every 16-dim m-tile md.
    float o[Gm::kMtDim][NTH][4];
    float m_run[NTH][2], l_run[NTH][2];
#pragma unroll
    for (int md = 0; md < Gm::kMtDim; ++md)
#pragma unroll
        for (int nh = 0; nh < NTH; ++nh) o[md][nh][0] = o[md][nh][1] = o[md][nh][2] = o[md][nh][3] = 0.f;
#pragma unroll
    for (int nh = 0; nh < NTH; ++nh) {
        m_run[nh][0] = m_run[nh][1] = -INFINITY;
        l_run[nh][0] = l_run[nh][1] = 0.f;
    }

    if (warp == kConsumerWarps) {
        // ================= producer warp =================
        if (lane == 0) {
            tma_prefetch_desc(&kmap);
            tma_prefetch_desc(&vmap);
        }
        const uint64_t pol = l2_policy_evict_first();
        const int32_t* table = a.block_tables + static_cast<size_t>(tseq) * a.max_blocks_per_seq + blk0;
        bool ok = true;
        int issued = 0;   // stages issued
        constexpr int kChunk = 32 / Gm::kBps * Gm::kBps;   // table entries per warp-wide load
        for (int j0 = 0; j0 < nblk && ok; j0 += kChunk) {
            const int jj = j0 + lane;
            int pid = 0;
            bool bad = false;
            if (lane < kChunk && jj < nblk) {
                pid = __ldg(table + jj);
                bad = pid < 0 || pid >= a.num_blocks;
            }
            if (__any_sync(0xffffffffu, bad) && lane == 0) {
                raise_error(a.err, PKV_DEVERR_BLOCK_ID);
                *s_abort = 1;
            }
            if (bad) pid = 0;   // load an in-range block; the output becomes NaN
            if (j0 == 0) pdl_wait();   // the pool may still be written by the previous kernel
            const int cnt = min(kChunk, nblk - j0);
            for (int i = 0; i < cnt; i += Gm::kBps) {
                const int js = (j0 + i) / Gm::kBps;   // stage index within the partition
                int pj[Gm::kBps];
#pragma unroll
                for (int b = 0; b < Gm::kBps; ++b) pj[b] = __shfl_sync(0xffffffffu, pid, (i + b) & 31);
                const int nb = min(Gm::kBps, cnt - i);
                const int stage = js % NST;
                if (lane == 0) {
                    if (js >= NST && !mbar_wait(bar_empty + 8 * stage, ((js / NST) - 1) & 1)) ok = false;
                    if (ok) {
                        const uint32_t fb = bar_full + 8 * stage;
                        const uint32_t sbase = base + stage * Gm::kStageBytes;
                        mbar_arrive_expect_tx(fb, 2 * nb * Gm::kTileBytes);
#pragma unroll
                        for (int b = 0; b < Gm::kBps; ++b) {
                            if (b < nb) {
#pragma unroll
                                for (int sub = 0; sub < Gm::kNsub; ++sub) {
                                    const uint32_t off = b * Gm::kTileBytes + sub * Gm::kSubBytes;
                                    tma_load_4d(sbase + off, &kmap, fb, sub * (128 / Gm::E), 0, kvh, pj[b], pol);
                                    tma_load_4d(sbase + Gm::kVOff + off, &vmap, fb, sub * (128 / Gm::E), 0, kvh, pj[b],
                                                pol);
                                }
                            }
                        }
                        issued = js + 1;
                    }
                }
                ok = __shfl_sync(0xffffffffu, ok, 0);
                if (!ok) break;
            }
        }
        if (lane == 0) {
            if (!ok) {
                raise_error(a.err, PKV_DEVERR_TIMEOUT);
                *s_abort = 1;
            }
            // no bulk copy may still be writing this CTA's shared memory when it moves on
            const uint64_t deadline = global_timer_ns() + kWaitLimitNs;
            for (int j = max(0, issued - NST); j < issued; ++j)
                if (!mbar_wait(bar_full + 8 * (j % NST), (j / NST) & 1, deadline)) {
                    raise_error(a.err, PKV_DEVERR_TIMEOUT);
                    break;
                }
        }
    } else {
        // ================= consumer warps =================
        const int r = lane >> 2, c = lane & 3;
        // Q^T fragments: B operand of S^T = K Q^T (k = head_dim, n = query head)
        uint32_t qb[Gm::kKsteps][NTH][2];
#pragma unroll
        for (int nh = 0; nh < NTH; ++nh) {
            const int hq = nh * 8 + r;
            const bool ok = hq < rows;
            const uint32_t* qrow = reinterpret_cast<const uint32_t*>(static_cast<const uint16_t*>(a.q) +
                                                                     row_of(ok ? hq : 0) * D);
            if constexpr (Gm::E == 1) {
                // permuted order: the lane's words of all k-steps are one 64-byte run of the row
                // (words 16c .. 16c + 15), so four 16-byte loads fetch them
                static_assert(Gm::kKsteps == 8, "E4M3 fragments assume head_dim 128");
                const uint4* q4 = reinterpret_cast<const uint4*>(qrow) + 4 * c;
                uint4 v[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) v[i] = ok ? __ldg(q4 + i) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
                for (int ks = 0; ks < Gm::kKsteps; ++ks) {
                    qb[ks][nh][0] = word(v[ks >> 1], 2 * (ks & 1));       // dims 32c + 4ks, +1
                    qb[ks][nh][1] = word(v[ks >> 1], 2 * (ks & 1) + 1);   // dims 32c + 4ks + 2, +3
                }
            } else {
#pragma unroll
                for (int ks = 0; ks < Gm::kKsteps; ++ks) {
                    const int d0 = Gm::qk_dim(c, ks);
                    qb[ks][nh][0] = ok ? __ldg(qrow + (d0 >> 1)) : 0u;
                    qb[ks][nh][1] = ok ? __ldg(qrow + ((d0 + Gm::kQkB1) >> 1)) : 0u;
                }
            }
        }
        pdl_wait();   // outputs and partials are written only after the previous kernel
        // per-lane ldmatrix row addresses (16-bit tiles): lane supplies row (lane & 7) of
        // matrix lane >> 3; the swizzle XOR only depends on (lane & 7)
        const int li = lane >> 3, l7 = lane & 7;
        const int k_tok = (li & 1) * 8 + l7;           // K: matrices (t0-7,k0-7) (t8-15,k0-7) (t0-7,k8-15) (t8-15,k8-15)
        const int k_hi = li >> 1;
        const int v_tok = (li >> 1) * 8 + l7;          // V^T: (d0-7,t0-7) (d8-15,t0-7) (d0-7,t8-15) (d8-15,t8-15)
        const int v_hi = li & 1;
        const float qk = a.qk_scale_log2;

        // stages per partition (a partition is a whole number of stages when a CTA holds several)
        const int spp = nlp > 1 ? PS / Gm::kStageTok : nstage;
        bool dead = false;   // a wait gave up: skip the remaining stages, still meet every barrier
        float* sm_o = reinterpret_cast<float*>(gbase + Gm::kRingBytes);      // [warps][rows][D]
        float* sm_m = sm_o + kConsumerWarps * Gm::kRowsMax * D;              // [warps][rows]
        float* sm_l = sm_m + kConsumerWarps * Gm::kRowsMax;                  // [warps][rows]
        for (int lp = 0; lp < nlp; ++lp) {
        const int s_lo = lp * spp, s_hi = min(nstage, s_lo + spp);
        for (int js = s_lo + (warp - s_lo % kConsumerWarps + kConsumerWarps) % kConsumerWarps; js < s_hi && !dead;
             js += kConsumerWarps) {
            const int stage = js % NST;
            const bool got = mbar_wait(bar_full + 8 * stage, (js / NST) & 1);
            if (!__all_sync(0xffffffffu, got)) {
                if (lane == 0) {
                    raise_error(a.err, PKV_DEVERR_TIMEOUT);
                    *s_abort = 1;
                }
                dead = true;
                break;
            }
            const uint32_t sb = base + stage * Gm::kStageBytes;
            const int valid = min(Gm::kStageTok, tok_end - (tok_begin + js * Gm::kStageTok));

            // ---- S^T = K Q^T  (M = 16 tokens, N = 8 heads, K = head_dim) ----
            float sc[Gm::kMtTok][NTH][4];
#pragma unroll
            for (int mt = 0; mt < Gm::kMtTok; ++mt)
#pragma unroll
                for (int nh = 0; nh < NTH; ++nh) sc[mt][nh][0] = sc[mt][nh][1] = sc[mt][nh][2] = sc[mt][nh][3] = 0.f;
            if constexpr (Gm::E == 2) {
#pragma unroll
                for (int ks = 0; ks < Gm::kKsteps; ++ks) {
#pragma unroll
                    for (int mt = 0; mt < Gm::kMtTok; ++mt) {
                        uint32_t ka[4];
                        ldsm_x4(ka, sb + Gm::at(mt * 16 + k_tok, 2 * ks + k_hi));
#pragma unroll
                        for (int nh = 0; nh < NTH; ++nh) mma16816<kBf16>(sc[mt][nh], ka, qb[ks][nh][0], qb[ks][nh][1]);
                    }
                }
            } else {
#pragma unroll
                for (int mt = 0; mt < Gm::kMtTok; ++mt) {
                    const int t0 = mt * 16 + r;
                    const uint4 x0 = lds128(sb + Gm::at(t0, 2 * c)), x1 = lds128(sb + Gm::at(t0, 2 * c + 1));
                    const uint4 y0 = lds128(sb + Gm::at(t0 + 8, 2 * c)), y1 = lds128(sb + Gm::at(t0 + 8, 2 * c + 1));
#pragma unroll
                    for (int ks = 0; ks < Gm::kKsteps; ++ks) {
                        const uint32_t wr = word(ks < 4 ? x0 : x1, ks & 3);   // token r, 4 bytes
                        const uint32_t wr8 = word(ks < 4 ? y0 : y1, ks & 3);  // token r + 8
                        uint32_t ka[4];
                        widen_e4m3x4<kBf16>(wr, ka[0], ka[2]);
                        widen_e4m3x4<kBf16>(wr8, ka[1], ka[3]);
#pragma unroll
                        for (int nh = 0; nh < NTH; ++nh) mma16816<kBf16>(sc[mt][nh], ka, qb[ks][nh][0], qb[ks][nh][1]);
                    }
                }
            }
            // ---- scale, mask, online softmax over the stage's tokens, per head ----
#pragma unroll
            for (int mt = 0; mt < Gm::kMtTok; ++mt)
#pragma unroll
                for (int nh = 0; nh < NTH; ++nh)
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int t = mt * 16 + r + (e >> 1) * 8;
                        const float x = sc[mt][nh][e] * qk;
                        sc[mt][nh][e] = t < valid ? x : -INFINITY;
                    }
            float alpha[NTH][2];
            bool rescale = false;
#pragma unroll
            for (int nh = 0; nh < NTH; ++nh)
#pragma unroll
                for (int hc = 0; hc < 2; ++hc) {
                    float mx = -INFINITY;
#pragma unroll
                    for (int mt = 0; mt < Gm::kMtTok; ++mt) mx = fmaxf(mx, fmaxf(sc[mt][nh][hc], sc[mt][nh][hc + 2]));
                    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
                    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
                    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
                    const float mnew = fmaxf(m_run[nh][hc], mx);
                    alpha[nh][hc] = ex2(m_run[nh][hc] - mnew);
                    rescale |= alpha[nh][hc] != 1.f;
                    m_run[nh][hc] = mnew;
                    float sum = 0.f;
#pragma unroll
                    for (int mt = 0; mt < Gm::kMtTok; ++mt) {
                        sc[mt][nh][hc] = ex2(sc[mt][nh][hc] - mnew);
                        sc[mt][nh][hc + 2] = ex2(sc[mt][nh][hc + 2] - mnew);
                        sum += sc[mt][nh][hc] + sc[mt][nh][hc + 2];
                    }
                    l_run[nh][hc] = l_run[nh][hc] * alpha[nh][hc] + sum;
                }
            if (__any_sync(0xffffffffu, rescale)) {
#pragma unroll
                for (int md = 0; md < Gm::kMtDim; ++md)
#pragma unroll
                    for (int nh = 0; nh < NTH; ++nh) {
                        o[md][nh][0] *= alpha[nh][0];
                        o[md][nh][1] *= alpha[nh][1];
                        o[md][nh][2] *= alpha[nh][0];
                        o[md][nh][3] *= alpha[nh][1];
                    }
            }
            // ---- P^T fragments (B operand of O^T = V^T P^T): transpose S^T's 8x8 blocks ----
            uint32_t pb[Gm::kMtTok][NTH][2], pl[Gm::kMtTok][NTH][2];
#pragma unroll
            for (int mt = 0; mt < Gm::kMtTok; ++mt)
#pragma unroll
                for (int nh = 0; nh < NTH; ++nh) {
                    pb[mt][nh][0] = movmatrix_t(pack2<kBf16>(sc[mt][nh][0], sc[mt][nh][1]));
                    pb[mt][nh][1] = movmatrix_t(pack2<kBf16>(sc[mt][nh][2], sc[mt][nh][3]));
                    if constexpr (kBf16) {
                        pl[mt][nh][0] = movmatrix_t(pack2<true>(bf16_residual(sc[mt][nh][0]), bf16_residual(sc[mt][nh][1])));
                        pl[mt][nh][1] = movmatrix_t(pack2<true>(bf16_residual(sc[mt][nh][2]), bf16_residual(sc[mt][nh][3])));
                    }
                }
            // ---- O^T += V^T P^T  (M = 16 head_dim rows, N = 8 heads, K = 16 tokens) ----
            const bool partial = valid < Gm::kStageTok;
            if constexpr (Gm::E == 2) {
#pragma unroll
                for (int mt = 0; mt < Gm::kMtTok; ++mt) {
                    const int t0 = mt * 16 + 2 * c;   // tokens of this lane's A halves: t0, t0+1 / t0+8, t0+9
#pragma unroll
                    for (int md = 0; md < Gm::kMtDim; ++md) {
                        uint32_t va[4];
                        ldsm_x4_trans(va, sb + Gm::kVOff + Gm::at(mt * 16 + v_tok, 2 * md + v_hi));
                        if (partial) {
                            va[0] = mask_pair(va[0], t0, valid);
                            va[1] = mask_pair(va[1], t0, valid);
                            va[2] = mask_pair(va[2], t0 + 8, valid);
                            va[3] = mask_pair(va[3], t0 + 8, valid);
                        }
#pragma unroll
                        for (int nh = 0; nh < NTH; ++nh) {
                            mma16816<kBf16>(o[md][nh], va, pb[mt][nh][0], pb[mt][nh][1]);
                            if constexpr (kBf16) mma16816<kBf16>(o[md][nh], va, pl[mt][nh][0], pl[mt][nh][1]);
                        }
                    }
                }
            } else {
#pragma unroll
                for (int mt = 0; mt < Gm::kMtTok; ++mt) {
                    const int t0 = mt * 16 + 2 * c;
                    uint4 v0 = lds128(sb + Gm::kVOff + Gm::at(t0, r));
                    uint4 v1 = lds128(sb + Gm::kVOff + Gm::at(t0 + 1, r));
                    uint4 v2 = lds128(sb + Gm::kVOff + Gm::at(t0 + 8, r));
                    uint4 v3 = lds128(sb + Gm::kVOff + Gm::at(t0 + 9, r));
                    if (partial) {
                        const uint4 z = make_uint4(0u, 0u, 0u, 0u);
                        if (t0 >= valid) v0 = z;
                        if (t0 + 1 >= valid) v1 = z;
                        if (t0 + 8 >= valid) v2 = z;
                        if (t0 + 9 >= valid) v3 = z;
                    }
#pragma unroll
                    for (int w = 0; w < 4; ++w) {
                        const uint32_t x0 = word(v0, w), x1 = word(v1, w), x2 = word(v2, w), x3 = word(v3, w);
                        // (dim d, token pair) bytes: d = 16r + 4w + {0,1} in e, {2,3} in f
                        const uint32_t e01 = __byte_perm(x0, x1, 0x5140u), e23 = __byte_perm(x2, x3, 0x5140u);
                        const uint32_t f01 = __byte_perm(x0, x1, 0x7362u), f23 = __byte_perm(x2, x3, 0x7362u);
                        uint32_t va[4], vb[4];
                        widen_e4m3x4<kBf16>(e01, va[0], va[1]);
                        widen_e4m3x4<kBf16>(e23, va[2], va[3]);
                        widen_e4m3x4<kBf16>(f01, vb[0], vb[1]);
                        widen_e4m3x4<kBf16>(f23, vb[2], vb[3]);
#pragma unroll
                        for (int nh = 0; nh < NTH; ++nh) {
                            mma16816<kBf16>(o[2 * w][nh], va, pb[mt][nh][0], pb[mt][nh][1]);
                            mma16816<kBf16>(o[2 * w + 1][nh], vb, pb[mt][nh][0], pb[mt][nh][1]);
                            if constexpr (kBf16) {
                                mma16816<kBf16>(o[2 * w][nh], va, pl[mt][nh][0], pl[mt][nh][1]);
                                mma16816<kBf16>(o[2 * w + 1][nh], vb, pl[mt][nh][0], pl[mt][nh][1]);
                            }
                        }
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_empty + 8 * stage);
        }
        // complete the per-head sums across the 8 lanes that share c
#pragma unroll
        for (int nh = 0; nh < NTH; ++nh)
#pragma unroll
            for (int hc = 0; hc < 2; ++hc) {
                float v = l_run[nh][hc];
                v += __shfl_xor_sync(0xffffffffu, v, 4);
                v += __shfl_xor_sync(0xffffffffu, v, 8);
                v += __shfl_xor_sync(0xffffffffu, v, 16);
                l_run[nh][hc] = v;
            }
        // ---- this partition's four warp states -> its output or partial (consumer warps only) ----
        {
            float* ow = sm_o + warp * Gm::kRowsMax * D;
#pragma unroll
            for (int md = 0; md < Gm::kMtDim; ++md)
#pragma unroll
                for (int nh = 0; nh < NTH; ++nh) {
                    const int h0 = nh * 8 + 2 * c;
                    const int d0 = Gm::o_dim(md, r), d1 = Gm::o_dim(md, r + 8);
                    ow[h0 * D + d0] = o[md][nh][0];
                    ow[(h0 + 1) * D + d0] = o[md][nh][1];
                    ow[h0 * D + d1] = o[md][nh][2];
                    ow[(h0 + 1) * D + d1] = o[md][nh][3];
                }
            if (r == 0) {
#pragma unroll
                for (int nh = 0; nh < NTH; ++nh)
#pragma unroll
                    for (int hc = 0; hc < 2; ++hc) {
                        sm_m[warp * Gm::kRowsMax + nh * 8 + 2 * c + hc] = m_run[nh][hc];
                        sm_l[warp * Gm::kRowsMax + nh * 8 + 2 * c + hc] = l_run[nh][hc];
                    }
            }
        }
        consumer_barrier();
        {
            if (lp == nlp - 1) pdl_trigger();   // the merge kernel (or the next step) may start its prologue
            const bool aborted = *s_abort != 0;
            const bool single = nparts == 1 && start == 0 && !prefix_pass;   // otherwise partials for the merge
            const float vs = a.v_scale;
            for (int e = threadIdx.x; e < rows * D; e += kConsumerWarps * 32) {
                const int hh = e / D, d = e - hh * D;
                float M = -INFINITY;
#pragma unroll
                for (int w = 0; w < kConsumerWarps; ++w) M = fmaxf(M, sm_m[w * Gm::kRowsMax + hh]);
                float num = 0.f, den = 0.f;
#pragma unroll
                for (int w = 0; w < kConsumerWarps; ++w) {
                    const float f = exp2f(sm_m[w * Gm::kRowsMax + hh] - M);
                    num += f * sm_o[(w * Gm::kRowsMax + hh) * D + d];
                    den += f * sm_l[w * Gm::kRowsMax + hh];
                }
                float val = num / den * vs;
                if (aborted) val = __int_as_float(0x7fc00000);
                if (single) {
                    store_out<kQBf16>(a.out, row_of(hh) * D + d, val);
                } else {
                    const size_t slot = row_of(hh) * a.max_partitions + a.slot_base + part0 + lp;
                    a.ws_o[slot * D + d] = val;
                    if (d == 0) a.ws_ml[slot] = make_float2(aborted ? __int_as_float(0x7fc00000) : M, den);
                }
            }
        }
        consumer_barrier();   // the buffer is rewritten by the next partition's states
        // fresh state for the next partition
#pragma unroll
        for (int md = 0; md < Gm::kMtDim; ++md)
#pragma unroll
            for (int nh = 0; nh < NTH; ++nh) o[md][nh][0] = o[md][nh][1] = o[md][nh][2] = o[md][nh][3] = 0.f;
#pragma unroll
        for (int nh = 0; nh < NTH; ++nh) {
            m_run[nh][0] = m_run[nh][1] = -INFINITY;
            l_run[nh][0] = l_run[nh][1] = 0.f;
        }
        }   // partitions of the CTA
    }
    if (warp == kConsumerWarps) pdl_trigger();   // the producer is done issuing
}

// ---- pass 2: merge partitions by log-sum-exp -------------------------------------

// One CTA of D threads per (sequence, query head): the partitions' (max, sum) pairs
// are staged in shared memory, the weights 2^(m_p - M) l_p computed once, and each
// thread (one head_dim element) sums its column with eight loads in flight.
template <bool kQBf16, int D>
__global__ void __launch_bounds__(D) decode_reduce_kernel(const DecodeArgs a) {
    extern __shared__ float sw[];   // [max_partitions] weights, then [D / 32] partial values
    pdl_trigger();
    pdl_wait();
    const int qh = blockIdx.x, s = blockIdx.y, d = threadIdx.x;
    const int L = __ldg(a.context_lens + s);
    const int PS = a.partition_size;
    // partials of a sequence: its prefix partitions in slots [0, np_pre) (shared-prefix
    // call only), then its own partitions from slot a.slot_base on
    const int start = a.seq_start ? __ldg(a.seq_start + s) : 0;
    const size_t row = static_cast<size_t>(s) * a.num_heads + qh;
    if (L < 0 || L > a.max_blocks_per_seq * a.block_size || L > a.max_context_len || start < 0 || start > L ||
        start % a.block_size != 0 || start > a.max_prefix_len) {
        if (start > 0) store_out<kQBf16>(a.out, row * D + d, __int_as_float(0x7fc00000));
        return;   // (a sequence without a prefix got its NaN from pass 1)
    }
    const int np_pre = start > 0 ? (start + a.prefix_partition_size - 1) / a.prefix_partition_size : 0;
    const int np_tail = (L - start + PS - 1) / PS;
    const int np = np_pre + np_tail;
    if (np_pre == 0 && np_tail <= 1) return;   // written by pass 1
    if (grid_timed_out(a.err)) {   // a pass gave up somewhere: its partials are not to be trusted
        store_out<kQBf16>(a.out, row * D + d, __int_as_float(0x7fc00000));
        return;
    }
    auto slot = [&](int p) { return p < np_pre ? p : a.slot_base + (p - np_pre); };
    const float2* ml = a.ws_ml + row * a.max_partitions;
    const float* wo = a.ws_o + row * a.max_partitions * D;
    if (np <= 8) {   // few partitions: every thread reads the pairs itself, all loads at once
        float2 v[8];
        float o[8];
#pragma unroll
        for (int p = 0; p < 8; ++p)
            if (p < np) {
                v[p] = ml[slot(p)];
                o[p] = wo[static_cast<size_t>(slot(p)) * D + d];
            }
        float M = -INFINITY;
#pragma unroll
        for (int p = 0; p < 8; ++p)
            if (p < np) {
                M = fmaxf(M, v[p].x);
                if (d == 0 && p < np_pre && __float_as_uint(v[p].y) == kUnwrittenSum)
                    raise_error(a.err, PKV_DEVERR_CONTEXT_LEN);   // no unit covered this prefix slot: NaN
            }
        float num = 0.f, den = 0.f;
#pragma unroll
        for (int p = 0; p < 8; ++p)
            if (p < np) {
                const float w = exp2f(v[p].x - M) * v[p].y;
                num += w * o[p];
                den += w;
            }
        store_out<kQBf16>(a.out, row * D + d, num / den);
        return;
    }
    float* red = sw + a.max_partitions;
    // M = max_p m_p
    float mx = -INFINITY;
    for (int p = d; p < np; p += D) mx = fmaxf(mx, ml[slot(p)].x);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    if ((d & 31) == 0) red[d >> 5] = mx;
    __syncthreads();
    float M = red[0];
#pragma unroll
    for (int w = 1; w < D / 32; ++w) M = fmaxf(M, red[w]);
    // weights and their sum
    float den = 0.f;
    for (int p = d; p < np; p += D) {
        const float2 v = ml[slot(p)];
        if (p < np_pre && __float_as_uint(v.y) == kUnwrittenSum) raise_error(a.err, PKV_DEVERR_CONTEXT_LEN);
        const float w = exp2f(v.x - M) * v.y;
        sw[p] = w;
        den += w;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
    __syncthreads();   // every thread has read red[] for M and written its weights
    if ((d & 31) == 0) red[d >> 5] = den;
    __syncthreads();
    float total = 0.f;
#pragma unroll
    for (int w = 0; w < D / 32; ++w) total += red[w];
    // weighted column sums, eight independent loads at a time
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    int p = 0;
    for (; p + 8 <= np; p += 8) {
        float o[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) o[i] = wo[static_cast<size_t>(slot(p + i)) * D + d];
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] += sw[p + i] * o[i];
    }
    for (; p < np; ++p) acc[0] += sw[p] * wo[static_cast<size_t>(slot(p)) * D + d];
    const float num = ((acc[0] + acc[1]) + (acc[2] + acc[3])) + ((acc[4] + acc[5]) + (acc[6] + acc[7]));
    store_out<kQBf16>(a.out, row * D + d, num / total);
}

// ---- host side -----------------------------------------------------------------------

// Automatic partition size: about 512 KB of K+V per (partition, KV head) -- 1,024
// tokens of 16-bit D=128, 2,048 of FP8 -- which measured best on the OPT-13B, GQA and
// long-context FP8 workloads (smaller partitions pay the cross-warp merge and the
// partials' round trip more often, larger ones starve the SMs); then halved (not
// below 4 blocks) while fewer than two work units per SM exist.
int pick_partition(int num_seqs, int num_kv_heads, int head_dim, int elem_bytes, int block_size,
                   int max_context_len, int requested) {
    const int cap = ((max_context_len > 0 ? max_context_len : 1) + block_size - 1) / block_size * block_size;
    if (requested > 0) return requested >= cap ? cap : requested;
    const int by_bytes = (512 * 1024) / (2 * head_dim * elem_bytes) / block_size * block_size;
    int p = by_bytes < cap ? by_bytes : cap;
    if (p < block_size) p = block_size;
    const long long target = 2LL * num_sms();
    const int floor_p = 4 * block_size;   // at least one block per consumer warp
    auto units = [&](int ps) {
        return static_cast<long long>(num_seqs) * num_kv_heads * ((cap + ps - 1) / ps);
    };
    while (p > floor_p && units(p) < target) {
        int np = (p / 2 + block_size - 1) / block_size * block_size;
        if (np < floor_p) np = floor_p;
        if (np == p) break;
        p = np;
    }
    return p;
}

bool encode_pool_map(CUtensorMap* map, const void* pool, int kv_dtype, int head_dim, int block_size,
                     int num_kv_heads, int num_blocks) {
    EncodeTiledFn enc = encode_tiled_fn();
    if (!enc) return false;
    const int e = kv_dtype == PKV_FP8_E4M3 ? 1 : 2;
    const cuuint64_t dims[4] = {static_cast<cuuint64_t>(head_dim), static_cast<cuuint64_t>(block_size),
                                static_cast<cuuint64_t>(num_kv_heads), static_cast<cuuint64_t>(num_blocks)};
    const cuuint64_t strides[3] = {static_cast<cuuint64_t>(head_dim) * e,
                                   static_cast<cuuint64_t>(block_size) * head_dim * e,
                                   static_cast<cuuint64_t>(num_kv_heads) * block_size * head_dim * e};
    const cuuint32_t box[4] = {static_cast<cuuint32_t>(128 / e), static_cast<cuuint32_t>(block_size), 1, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    return enc(map, e == 1 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_UINT16, 4,
               const_cast<void*>(pool), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
               CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int KV, bool kQBf16, int D, int BS, bool kHi>
pkv_status launch_pass1(const DecodeArgs& a, const CUtensorMap& km, const CUtensorMap& vm, unsigned gx, unsigned gz,
                        cudaStream_t st) {
    using Gm = Geo<KV, D, BS, kHi>;
    auto kern = paged_decode_kernel<KV, kQBf16, D, BS, kHi>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Gm::kSmemBytes) != cudaSuccess)
        return PKV_ERR_CUDA;
    const dim3 grid(static_cast<unsigned>(a.num_kv_heads), gz, gx);
    return launch_pdl(kern, grid, dim3(kThreads), Gm::kSmemBytes, st, a, km, vm) == cudaSuccess ? PKV_OK
                                                                                                : PKV_ERR_CUDA;
}

template <bool kQBf16, int D>
pkv_status launch_merge(const DecodeArgs& a, cudaStream_t st) {
    const size_t rsmem = (static_cast<size_t>(a.max_partitions) + D / 32) * sizeof(float);
    auto rk = decode_reduce_kernel<kQBf16, D>;
    if (rsmem > 48 * 1024 &&
        cudaFuncSetAttribute(rk, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(rsmem)) != cudaSuccess)
        return PKV_ERR_CUDA;
    return launch_pdl(rk, dim3(a.num_heads, a.num_seqs), dim3(D), rsmem, st, a) == cudaSuccess ? PKV_OK
                                                                                               : PKV_ERR_CUDA;
}

struct Pass1 {
    const DecodeArgs& a;
    const CUtensorMap& km;
    const CUtensorMap& vm;
    unsigned gx, gz;
    cudaStream_t st;
    template <int KV, bool QB, int D, int BS, bool HI>
    pkv_status run() const { return launch_pass1<KV, QB, D, BS, HI>(a, km, vm, gx, gz, st); }
};

struct Merge {
    const DecodeArgs& a;
    cudaStream_t st;
    template <int KV, bool QB, int D, int BS, bool HI>
    pkv_status run() const { return launch_merge<QB, D>(a, st); }
};

template <int KV, bool QB, int D, class F>
pkv_status with_bs(int bs, bool hi, const F& f) {
    if (bs == 16) return hi ? f.template run<KV, QB, D, 16, true>() : f.template run<KV, QB, D, 16, false>();
    return hi ? f.template run<KV, QB, D, 32, true>() : f.template run<KV, QB, D, 32, false>();
}

// Calls f.run<...>() for the kernel instance of these (validated) arguments.
template <class F>
pkv_status with_instance(pkv_dtype kv, pkv_dtype qd, int D, int bs, bool hi, const F& f) {
    switch (kv) {
    case PKV_F16:
        return D == 64 ? with_bs<KV_F16, false, 64>(bs, hi, f) : with_bs<KV_F16, false, 128>(bs, hi, f);
    case PKV_BF16:
        return D == 64 ? with_bs<KV_BF16, true, 64>(bs, hi, f) : with_bs<KV_BF16, true, 128>(bs, hi, f);
    case PKV_FP8_E4M3:
        return qd == PKV_BF16 ? with_bs<KV_E4M3, true, 128>(bs, hi, f) : with_bs<KV_E4M3, false, 128>(bs, hi, f);
    }
    return PKV_ERR_UNSUPPORTED;
}

// Checks shared by the decode entry points (host-visible arguments only).
pkv_status validate(const void* out, const void* q, pkv_dtype q_dtype, const void* k_pool, const void* v_pool,
                    pkv_dtype kv_dtype, float k_scale, float v_scale, const int32_t* block_tables,
                    int max_blocks_per_seq, const int32_t* context_lens, int max_context_len, int num_seqs,
                    int num_heads, int num_kv_heads, int head_dim, int block_size, int num_blocks, float scale,
                    int partition_size) {
    if (num_seqs < 0 || num_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 ||
        num_blocks <= 0 || max_blocks_per_seq <= 0 || max_context_len < 0 || partition_size < 0)
        return PKV_ERR_INVALID_ARG;
    if (num_heads % num_kv_heads != 0) return PKV_ERR_INVALID_ARG;
    if (!std::isfinite(scale)) return PKV_ERR_INVALID_ARG;
    if (num_heads / num_kv_heads > 16) return PKV_ERR_UNSUPPORTED;
    if (block_size != 16 && block_size != 32) return PKV_ERR_UNSUPPORTED;
    if (partition_size % block_size != 0) return PKV_ERR_INVALID_ARG;
    if (q_dtype != PKV_F16 && q_dtype != PKV_BF16) return PKV_ERR_UNSUPPORTED;
    if (kv_dtype != q_dtype && kv_dtype != PKV_FP8_E4M3) return PKV_ERR_UNSUPPORTED;
    if (kv_dtype == PKV_FP8_E4M3) {
        if (head_dim != 128) return PKV_ERR_UNSUPPORTED;
        if (!(k_scale > 0.f && v_scale > 0.f) || !std::isfinite(k_scale) || !std::isfinite(v_scale))
            return PKV_ERR_INVALID_ARG;
    } else if (head_dim != 64 && head_dim != 128) {
        return PKV_ERR_UNSUPPORTED;
    }
    if (num_seqs > 65535 || num_kv_heads > 65535) return PKV_ERR_UNSUPPORTED;
    if (num_seqs == 0) return PKV_OK;
    if (!out || !q || !k_pool || !v_pool || !block_tables || !context_lens) return PKV_ERR_INVALID_ARG;
    if (!aligned16(out) || !aligned16(q) || !aligned16(k_pool) || !aligned16(v_pool) ||
        (reinterpret_cast<uintptr_t>(block_tables) & 3) || (reinterpret_cast<uintptr_t>(context_lens) & 3))
        return PKV_ERR_ALIGNMENT;
    return PKV_OK;
}

DecodeArgs base_args(void* out, const void* q, const int32_t* block_tables, int max_blocks_per_seq,
                     const int32_t* context_lens, int max_context_len, int num_seqs, int num_heads,
                     int num_kv_heads, int num_blocks, int block_size, pkv_dtype kv_dtype, float k_scale,
                     float v_scale, float scale, int ps, uint32_t* device_error) {
    DecodeArgs a{};
    a.out = out;
    a.q = q;
    a.block_tables = block_tables;
    a.context_lens = context_lens;
    a.err = device_error;
    a.max_blocks_per_seq = max_blocks_per_seq;
    a.max_context_len = max_context_len;
    a.num_seqs = num_seqs;
    a.num_heads = num_heads;
    a.num_kv_heads = num_kv_heads;
    a.num_blocks = num_blocks;
    a.block_size = block_size;
    a.partition_size = ps;
    a.parts_per_cta = 1;
    const float ks = kv_dtype == PKV_FP8_E4M3 ? k_scale : 1.f;
    a.qk_scale_log2 = static_cast<float>(static_cast<double>(scale) * ks * 1.4426950408889634);
    a.v_scale = kv_dtype == PKV_FP8_E4M3 ? v_scale : 1.f;
    return a;
}

// Tokens of one ring stage of the decode kernel (the Geo rule: a stage moves at least 8 KB).
int stage_tokens(pkv_dtype kv_dtype, int head_dim, int block_size) {
    const int tile = block_size * head_dim * (kv_dtype == PKV_FP8_E4M3 ? 1 : 2);
    const int bps = 2 * tile >= 8192 ? 1 : 8192 / (2 * tile);
    return bps * block_size;
}

// Partitions one CTA streams: a stated partition size smaller than the automatic choice keeps its
// partials (one per stated partition, merged exactly), but a CTA takes as many consecutive ones as
// the automatic size holds, so that the ring streams across them instead of starting again.
int partitions_per_cta(int ps, int num_seqs, int num_kv_heads, int head_dim, pkv_dtype kv_dtype, int block_size,
                       int max_context_len, int requested) {
    if (requested <= 0) return 1;
    const int auto_ps = pick_partition(num_seqs, num_kv_heads, head_dim, kv_dtype == PKV_FP8_E4M3 ? 1 : 2,
                                       block_size, max_context_len, 0);
    if (auto_ps <= ps || ps % stage_tokens(kv_dtype, head_dim, block_size) != 0) return 1;
    return auto_ps / ps;
}

size_t partials_bytes(size_t rows, int head_dim) {
    return (rows * head_dim * sizeof(float) + 255) / 256 * 256 + rows * sizeof(float2);
}

void set_partials(DecodeArgs& a, void* workspace, size_t rows, int head_dim) {
    a.ws_o = static_cast<float*>(workspace);
    a.ws_ml = reinterpret_cast<float2*>(static_cast<uint8_t*>(workspace) +
                                        (rows * head_dim * sizeof(float) + 255) / 256 * 256);
}

}  // namespace
}  // namespace pkv

extern "C" int pkv_decode_partition_size(int num_seqs, int num_kv_heads, int head_dim, pkv_dtype kv_dtype,
                                         int block_size, int max_context_len, int partition_size) {
    if (num_seqs < 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 || max_context_len < 0 ||
        partition_size < 0 || partition_size % block_size != 0)
        return 0;
    const int e = kv_dtype == PKV_FP8_E4M3 ? 1 : 2;
    return pkv::pick_partition(num_seqs, num_kv_heads, head_dim, e, block_size, max_context_len, partition_size);
}

extern "C" size_t pkv_decode_workspace_bytes(int num_seqs, int num_heads, int num_kv_heads, int head_dim,
                                             pkv_dtype kv_dtype, int block_size, int max_context_len,
                                             int partition_size) {
    const int ps = pkv_decode_partition_size(num_seqs, num_kv_heads, head_dim, kv_dtype, block_size,
                                             max_context_len, partition_size);
    if (ps <= 0 || num_heads <= 0 || head_dim <= 0) return 0;
    const long long parts = (static_cast<long long>(max_context_len) + ps - 1) / ps;
    if (parts <= 1) return 0;
    return pkv::partials_bytes(static_cast<size_t>(num_seqs) * num_heads * static_cast<size_t>(parts), head_dim);
}

extern "C" pkv_status pkv_paged_attn_decode(void* out, const void* q, pkv_dtype q_dtype, const void* k_pool,
                                            const void* v_pool, pkv_dtype kv_dtype, float k_scale, float v_scale,
                                            const int32_t* block_tables, int max_blocks_per_seq,
                                            const int32_t* context_lens, int max_context_len, int num_seqs,
                                            int num_heads, int num_kv_heads, int head_dim, int block_size,
                                            int num_blocks, float scale, int partition_size, void* workspace,
                                            size_t workspace_bytes, uint32_t* device_error, void* stream) {
    using namespace pkv;
    const pkv_status v = validate(out, q, q_dtype, k_pool, v_pool, kv_dtype, k_scale, v_scale, block_tables,
                                  max_blocks_per_seq, context_lens, max_context_len, num_seqs, num_heads,
                                  num_kv_heads, head_dim, block_size, num_blocks, scale, partition_size);
    if (v != PKV_OK || num_seqs == 0) return v;
    const int ps = pick_partition(num_seqs, num_kv_heads, head_dim, kv_dtype == PKV_FP8_E4M3 ? 1 : 2, block_size,
                                  max_context_len, partition_size);
    const int parts = max_context_len > 0 ? (max_context_len + ps - 1) / ps : 1;
    const size_t need = pkv_decode_workspace_bytes(num_seqs, num_heads, num_kv_heads, head_dim, kv_dtype,
                                                   block_size, max_context_len, partition_size);
    if (need > 0 && (!workspace || workspace_bytes < need)) return PKV_ERR_WORKSPACE;
    if (need > 0 && (reinterpret_cast<uintptr_t>(workspace) & 255)) return PKV_ERR_ALIGNMENT;

    DecodeArgs a = base_args(out, q, block_tables, max_blocks_per_seq, context_lens, max_context_len, num_seqs,
                             num_heads, num_kv_heads, num_blocks, block_size, kv_dtype, k_scale, v_scale, scale, ps,
                             device_error);
    a.max_partitions = parts;
    a.parts_per_cta = partitions_per_cta(ps, num_seqs, num_kv_heads, head_dim, kv_dtype, block_size, max_context_len,
                                         partition_size);
    if (need) set_partials(a, workspace, static_cast<size_t>(num_seqs) * num_heads * parts, head_dim);

    alignas(64) CUtensorMap km;
    alignas(64) CUtensorMap vm;
    if (!encode_pool_map(&km, k_pool, kv_dtype, head_dim, block_size, num_kv_heads, num_blocks) ||
        !encode_pool_map(&vm, v_pool, kv_dtype, head_dim, block_size, num_kv_heads, num_blocks))
        return PKV_ERR_CUDA;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const bool hi = num_heads / num_kv_heads > 8;
    const unsigned groups = static_cast<unsigned>((parts + a.parts_per_cta - 1) / a.parts_per_cta);
    pkv_status r = with_instance(kv_dtype, q_dtype, head_dim, block_size, hi,
                                 Pass1{a, km, vm, groups, static_cast<unsigned>(num_seqs), st});
    if (r == PKV_OK && parts > 1) r = with_instance(kv_dtype, q_dtype, head_dim, block_size, hi, Merge{a, st});
    return r;
}

// ---- shared-prefix decode -----------------------------------------------------------------

namespace pkv {
namespace {
// The prefix pass is partitioned on its own: it has one work unit per (unit, KV head)
// and partition, so its partitions shrink until the SMs have enough of them.
//
// Automatic choice: a whole prefix per CTA needs no merge of prefix partitions, so a prefix is only
// split while the (unit, KV head) pairs would leave more than a quarter of the CTA slots empty.  The
// slots are those of the 16-row instance (two CTAs per SM), which units of 16 / G sequences use.
int prefix_partition(int num_units, int num_kv_heads, int head_dim, pkv_dtype kv_dtype, int block_size,
                     int max_prefix_len, int partition_size) {
    if (max_prefix_len <= 0) return block_size;
    if (partition_size > 0)
        return pkv_decode_partition_size(num_units > 0 ? num_units : 1, num_kv_heads, head_dim, kv_dtype,
                                         block_size, max_prefix_len, partition_size);
    const long long slots = 2LL * num_sms();
    const long long pairs = static_cast<long long>(num_units > 0 ? num_units : 1) * num_kv_heads;
    const int nblk = (max_prefix_len + block_size - 1) / block_size;
    const int max_split = nblk / 4 > 1 ? nblk / 4 : 1;   // at least four blocks per partition
    int k = 1;
    while (k < max_split && pairs * k * 4 < slots * 3) ++k;
    return (nblk + k - 1) / k * block_size;
}
}  // namespace
}  // namespace pkv

extern "C" size_t pkv_shared_prefix_workspace_bytes(int num_seqs, int num_heads, int num_kv_heads, int head_dim,
                                                    pkv_dtype kv_dtype, int block_size, int max_context_len,
                                                    int num_units, int max_prefix_len, int partition_size) {
    const int ps = pkv_decode_partition_size(num_seqs, num_kv_heads, head_dim, kv_dtype, block_size,
                                             max_context_len, partition_size);
    if (ps <= 0 || num_heads <= 0 || head_dim <= 0 || max_prefix_len < 0 || max_prefix_len > max_context_len)
        return 0;
    const int ps_pre = pkv::prefix_partition(num_units, num_kv_heads, head_dim, kv_dtype, block_size, max_prefix_len,
                                             partition_size);
    if (ps_pre <= 0) return 0;
    const int parts = (max_prefix_len + ps_pre - 1) / ps_pre + (max_context_len + ps - 1) / ps;
    return pkv::partials_bytes(static_cast<size_t>(num_seqs) * num_heads * static_cast<size_t>(parts), head_dim);
}

// Automatic plan: when the shared prefixes, counted once per unit, fit in L2, the plain call's
// repeated reads of them are L2 hits and its single pass beats the tail pass + prefix pass +
// merge, so the plain call runs.
extern "C" int pkv_shared_prefix_plan_used(int num_units, int num_kv_heads, int head_dim, pkv_dtype kv_dtype,
                                           int max_prefix_len, int plan) {
    if (plan != PKV_PREFIX_PLAN_AUTO && plan != PKV_PREFIX_PLAN_SHARED && plan != PKV_PREFIX_PLAN_PLAIN) return -1;
    if (plan == PKV_PREFIX_PLAN_PLAIN || num_units <= 0 || max_prefix_len <= 0) return PKV_PREFIX_PLAN_PLAIN;
    if (plan == PKV_PREFIX_PLAN_SHARED) return PKV_PREFIX_PLAN_SHARED;
    const double per_token = 2.0 * num_kv_heads * head_dim * (kv_dtype == PKV_FP8_E4M3 ? 1 : 2);
    return static_cast<double>(num_units) * max_prefix_len * per_token > static_cast<double>(pkv::l2_bytes())
               ? PKV_PREFIX_PLAN_SHARED
               : PKV_PREFIX_PLAN_PLAIN;
}

extern "C" pkv_status pkv_paged_attn_decode_shared_prefix(
    void* out, const void* q, pkv_dtype q_dtype, const void* k_pool, const void* v_pool, pkv_dtype kv_dtype,
    float k_scale, float v_scale, const int32_t* block_tables, int max_blocks_per_seq, const int32_t* context_lens,
    int max_context_len, int num_seqs, int num_heads, int num_kv_heads, int head_dim, int block_size,
    int num_blocks, float scale, int partition_size, const int32_t* seq_prefix_len, const int32_t* unit_seqs,
    const int32_t* unit_len, int num_units, int unit_width, int max_prefix_len, int plan, void* workspace,
    size_t workspace_bytes, uint32_t* device_error, void* stream) {
    using namespace pkv;
    const pkv_status v = validate(out, q, q_dtype, k_pool, v_pool, kv_dtype, k_scale, v_scale, block_tables,
                                  max_blocks_per_seq, context_lens, max_context_len, num_seqs, num_heads,
                                  num_kv_heads, head_dim, block_size, num_blocks, scale, partition_size);
    if (v != PKV_OK || num_seqs == 0) return v;
    const int G = num_heads / num_kv_heads;
    if (num_units < 0 || num_units > 65535 || unit_width <= 0 || max_prefix_len < 0 ||
        max_prefix_len > max_context_len || max_prefix_len % block_size != 0 ||
        (plan != PKV_PREFIX_PLAN_AUTO && plan != PKV_PREFIX_PLAN_SHARED && plan != PKV_PREFIX_PLAN_PLAIN))
        return PKV_ERR_INVALID_ARG;
    if (unit_width * G > 16) return PKV_ERR_UNSUPPORTED;
    if (!seq_prefix_len || (num_units > 0 && (!unit_seqs || !unit_len))) return PKV_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(seq_prefix_len) & 3) || (reinterpret_cast<uintptr_t>(unit_seqs) & 3) ||
        (reinterpret_cast<uintptr_t>(unit_len) & 3))
        return PKV_ERR_ALIGNMENT;
    const int ps = pick_partition(num_seqs, num_kv_heads, head_dim, kv_dtype == PKV_FP8_E4M3 ? 1 : 2, block_size,
                                  max_context_len, partition_size);
    const int ps_pre = prefix_partition(num_units, num_kv_heads, head_dim, kv_dtype, block_size, max_prefix_len,
                                        partition_size);
    const int p_pre = (max_prefix_len + ps_pre - 1) / ps_pre;
    const int p_tail = max_context_len > 0 ? (max_context_len + ps - 1) / ps : 1;
    const size_t need = pkv_shared_prefix_workspace_bytes(num_seqs, num_heads, num_kv_heads, head_dim, kv_dtype,
                                                          block_size, max_context_len, num_units, max_prefix_len,
                                                          partition_size);
    if (!workspace || workspace_bytes < need) return PKV_ERR_WORKSPACE;
    if (reinterpret_cast<uintptr_t>(workspace) & 255) return PKV_ERR_ALIGNMENT;

    // the plain call's workspace is never larger than this one's
    if (pkv_shared_prefix_plan_used(num_units, num_kv_heads, head_dim, kv_dtype, max_prefix_len, plan) !=
        PKV_PREFIX_PLAN_SHARED)
        return pkv_paged_attn_decode(out, q, q_dtype, k_pool, v_pool, kv_dtype, k_scale, v_scale, block_tables,
                                     max_blocks_per_seq, context_lens, max_context_len, num_seqs, num_heads,
                                     num_kv_heads, head_dim, block_size, num_blocks, scale, partition_size,
                                     workspace, workspace_bytes, device_error, stream);

    DecodeArgs a = base_args(out, q, block_tables, max_blocks_per_seq, context_lens, max_context_len, num_seqs,
                             num_heads, num_kv_heads, num_blocks, block_size, kv_dtype, k_scale, v_scale, scale, ps,
                             device_error);
    a.max_partitions = p_pre + p_tail;
    a.max_prefix_len = max_prefix_len;
    a.prefix_partition_size = ps_pre;
    set_partials(a, workspace, static_cast<size_t>(num_seqs) * num_heads * a.max_partitions, head_dim);

    alignas(64) CUtensorMap km;
    alignas(64) CUtensorMap vm;
    if (!encode_pool_map(&km, k_pool, kv_dtype, head_dim, block_size, num_kv_heads, num_blocks) ||
        !encode_pool_map(&vm, v_pool, kv_dtype, head_dim, block_size, num_kv_heads, num_blocks))
        return PKV_ERR_CUDA;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    // The tail pass runs first: it also marks every prefix slot a merge will read, so that the
    // prefix pass (next) leaves the marker only where no unit covers a sequence's prefix.
    DecodeArgs at = a;   // each sequence's own tokens, from the end of its prefix
    at.seq_start = seq_prefix_len;
    at.slot_base = p_pre;
    pkv_status r = with_instance(kv_dtype, q_dtype, head_dim, block_size, G > 8,
                                 Pass1{at, km, vm, static_cast<unsigned>(p_tail), static_cast<unsigned>(num_seqs), st});
    if (r == PKV_OK) {   // shared tokens: every unit's rows against its prefix, once
        DecodeArgs ap = a;
        ap.partition_size = ps_pre;
        ap.seq_start = seq_prefix_len;   // read only to check the members' prefix lengths
        ap.unit_seqs = unit_seqs;
        ap.unit_len = unit_len;
        ap.unit_width = unit_width;
        ap.slot_base = 0;
        r = with_instance(kv_dtype, q_dtype, head_dim, block_size, unit_width * G > 8,
                          Pass1{ap, km, vm, static_cast<unsigned>(p_pre), static_cast<unsigned>(num_units), st});
    }
    if (r == PKV_OK) r = with_instance(kv_dtype, q_dtype, head_dim, block_size, G > 8, Merge{at, st});
    return r;
}

// ---- decode with a library-owned workspace (no allocation by the caller) ------------
//
// For callers that cannot call cudaMalloc: code that runs where every device
// allocation must go through someone else's allocator (a host framework that
// owns the device memory budget), or a serving loop that must not allocate
// after start-up because cudaMalloc can synchronise the device and stall.
// The split-context workspace then lives in this file-scope device array,
// which every GPU that loads the library holds until the process exits.
// Host code cannot use the array's name as a device address (it names a
// host-side stand-in), so each device's address is looked up once with
// cudaGetSymbolAddress, with that device current, on the first call made on
// that device; make that first call before any stream capture.  The address
// is kept for the life of the process: it does not survive cudaDeviceReset
// (which unloads the module), so do not use this call after one.

namespace pkv {
namespace {

constexpr size_t kStaticWsBytes = 64ull << 20;   // PKV_STATIC_WORKSPACE_BYTES
static __device__ __align__(256) uint8_t g_static_ws[kStaticWsBytes];

constexpr int kMaxDevices = 64;
std::mutex g_static_ws_mu;
void* g_static_ws_ptr[kMaxDevices] = {};

// Device address of g_static_ws on the current device (set up once per device).
cudaError_t static_ws_address(void** ptr) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_static_ws_mu);
    if (!g_static_ws_ptr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_static_ws);
        if (e != cudaSuccess) return e;
        g_static_ws_ptr[dev] = p;
    }
    *ptr = g_static_ws_ptr[dev];
    return cudaSuccess;
}

}  // namespace
}  // namespace pkv

static_assert(pkv::kStaticWsBytes == PKV_STATIC_WORKSPACE_BYTES, "header and library disagree");

extern "C" pkv_status pkv_paged_attn_decode_static_ws(
    void* out, const void* q, pkv_dtype q_dtype, const void* k_pool, const void* v_pool, pkv_dtype kv_dtype,
    float k_scale, float v_scale, const int32_t* block_tables, int max_blocks_per_seq,
    const int32_t* context_lens, int max_context_len, int num_seqs, int num_heads, int num_kv_heads,
    int head_dim, int block_size, int num_blocks, float scale, int partition_size, uint32_t* device_error,
    void* stream) {
    const pkv_status v = pkv::validate(out, q, q_dtype, k_pool, v_pool, kv_dtype, k_scale, v_scale, block_tables,
                                       max_blocks_per_seq, context_lens, max_context_len, num_seqs, num_heads,
                                       num_kv_heads, head_dim, block_size, num_blocks, scale, partition_size);
    if (v != PKV_OK || num_seqs == 0) return v;
    const size_t need = pkv_decode_workspace_bytes(num_seqs, num_heads, num_kv_heads, head_dim, kv_dtype,
                                                   block_size, max_context_len, partition_size);
    if (need > pkv::kStaticWsBytes) return PKV_ERR_WORKSPACE;
    void* ws = nullptr;
    if (need > 0 && pkv::static_ws_address(&ws) != cudaSuccess) return PKV_ERR_CUDA;
    return pkv_paged_attn_decode(out, q, q_dtype, k_pool, v_pool, kv_dtype, k_scale, v_scale, block_tables,
                                 max_blocks_per_seq, context_lens, max_context_len, num_seqs, num_heads,
                                 num_kv_heads, head_dim, block_size, num_blocks, scale, partition_size, ws,
                                 need > 0 ? pkv::kStaticWsBytes : 0, device_error, stream);
}
