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
//   * Work unit = (partition of <= partition_size tokens, KV head, sequence):
//     one CTA.  All G query heads of the KV head ride in the same CTA, so each
//     K/V tile crosses HBM once per group (GQA; glossary "PagedAttention",
//     section "Related methods").
//   * One producer warp issues TMA tile loads.  The pool is described to TMA
//     as a 4-D tensor [head_dim, block_size, num_kv_heads, num_blocks]; the
//     block-table indirection is simply the outermost tile coordinate.  Tiles
//     land in shared memory with 128-byte swizzling, in a ring of stages
//     guarded by transaction barriers (full: TMA bytes arrived; empty:
//     consumer done), with evict-first L2 hints since the KV is streamed once.
//   * Four consumer warps take blocks round-robin.  Each computes
//     S = Q K^T for its block with mma.sync m16n8k16 (query heads as M,
//     padded to 16; tokens as N; head_dim as K), an online softmax in
//     registers (running max and sum, base-2 exponent), and O += P V with the
//     P fragments taken straight from the S accumulators.  FP8 E4M3 tiles are
//     widened to f16 (or bf16) in registers, two values per instruction, so
//     the MMA sees exact values and no dequantised copy is written anywhere.
//   * Operand fragments are read with 16-byte shared loads.  The head_dim
//     axis of the QK contraction and the output-column axis of PV are
//     permuted (the same permutation on both operands, undone on output) so
//     that each thread's fragment comes from contiguous bytes, and with the
//     swizzle every 8-lane phase touches 8 distinct bank groups.
//   * The four warps' partial states are merged in shared memory; a CTA that
//     covers its whole sequence writes the output, otherwise it writes
//     (max, sum, normalised output) to the workspace and a second small
//     kernel merges the partitions.
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
};

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

// Two E4M3 values (low byte first) -> two MMA operands packed in 32 bits (exact).
template <bool kBf16>
__device__ __forceinline__ uint32_t widen_e4m3x2(uint32_t two_bytes) {
    const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(two_bytes & 0xffffu),
                                                     __NV_E4M3);
    if constexpr (!kBf16) {
        return static_cast<uint32_t>(h.x) | (static_cast<uint32_t>(h.y) << 16);
    } else {
        const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&h));
        const __nv_bfloat162 b = __floats2bfloat162_rn(f.x, f.y);
        return *reinterpret_cast<const uint32_t*>(&b);
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

template <int KV, int D, int BS>
struct Geo {
    static constexpr int E = KV == KV_E4M3 ? 1 : 2;   // element bytes
    static constexpr int kNsub = D * E / 128;          // 128-byte sub-rows per token row
    static constexpr int kSubBytes = BS * 128;         // one swizzled sub-tile
    static constexpr int kTileBytes = kNsub * kSubBytes;
    static constexpr int kStageBytes = 2 * kTileBytes; // K tile + V tile
    static constexpr int kDpc = 16 / E;                // elements per 16-byte chunk
    static constexpr int kKsteps = D / 16;             // k-steps of the QK contraction
    static constexpr int kKpc = 4 / E;                 // QK k-steps served by one chunk
    static constexpr int kNtS = BS / 8;                // score n-tiles per block
    static constexpr int kKkPV = BS / 16;              // PV k-steps per block
    static constexpr int kNtO = D / 8;                 // output n-tiles
    static constexpr int kStages = (65536 / kStageBytes) < 4 ? 4 : ((65536 / kStageBytes) > 16 ? 16 : (65536 / kStageBytes));
    static constexpr int kRingBytes = kStages * kStageBytes;
    static constexpr int kMergeBytes = kConsumerWarps * 16 * (D + 2) * 4;
    static constexpr int kDataBytes = kRingBytes > kMergeBytes ? kRingBytes : kMergeBytes;
    static constexpr int kSmemBytes = 1024 /* alignment slack */ + kDataBytes + kStages * 16 + 16;
    static_assert(D * E == 128 || D * E == 256, "row must be 128 or 256 bytes");
    static_assert(kStages % kConsumerWarps == 0, "stage -> warp mapping must be fixed");

    // First head_dim index of the 4 consecutive elements a thread with quad
    // index c feeds into QK k-step ks (b0 covers base, base+1; b1 base+2, base+3).
    __device__ static __forceinline__ int k_base(int c, int ks) {
        const int qc = ks / kKpc, sub = qc >> 1, i = qc & 1;
        const int w0 = (ks % kKpc) * E;                  // first 32-bit word of the k-step
        return sub * (128 / E) + (2 * c + i) * kDpc + w0 * (4 / E);
    }
    // head_dim index of output column `col` (0..7) of PV n-tile nt.
    __device__ static __forceinline__ int o_dim(int nt, int col) {
        const int sub = nt / kDpc, dd = nt % kDpc;
        return sub * (128 / E) + col * kDpc + dd;
    }
};

// ---- pass 1: one CTA per (partition, KV head, sequence) ------------------------------

template <int KV, bool kQBf16, int D, int BS, bool kHi>
__global__ void __launch_bounds__(kThreads)
paged_decode_kernel(const DecodeArgs a, const __grid_constant__ CUtensorMap kmap,
                    const __grid_constant__ CUtensorMap vmap) {
    using Gm = Geo<KV, D, BS>;
    constexpr bool kBf16 = (KV == KV_BF16) || (KV == KV_E4M3 && kQBf16);
    constexpr int NST = Gm::kStages;

    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_addr(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* gbase = smem_raw + (base - raw);
    const uint32_t bar_full = base + Gm::kDataBytes;
    const uint32_t bar_empty = bar_full + NST * 8;
    volatile int* s_abort = reinterpret_cast<volatile int*>(gbase + Gm::kDataBytes + NST * 16);

    const int part = blockIdx.x, kvh = blockIdx.y, s = blockIdx.z;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = a.num_heads / a.num_kv_heads;
    const int H = a.num_heads;
    const int L = __ldg(a.context_lens + s);
    const size_t out_row0 = static_cast<size_t>(s) * H + static_cast<size_t>(kvh) * G;

    const bool bad_len = L < 0 || L > a.max_blocks_per_seq * BS || L > a.max_context_len;
    const bool give_up = grid_timed_out(a.err);
    if (bad_len || L == 0 || give_up) {
        if (part == 0) {
            if (bad_len && threadIdx.x == 0) raise_error(a.err, PKV_DEVERR_CONTEXT_LEN);
            const float v = (bad_len || give_up) ? __int_as_float(0x7fc00000) : 0.f;
            for (int e = threadIdx.x; e < G * D; e += kThreads)
                store_out<kQBf16>(a.out, out_row0 * D + e, v);
        }
        return;
    }
    const int PS = a.partition_size;
    const int nparts = (L + PS - 1) / PS;
    if (part >= nparts) return;
    const int tok_begin = part * PS;
    const int tok_end = min(L, tok_begin + PS);
    const int nblk = (tok_end - tok_begin + BS - 1) / BS;
    const int blk0 = tok_begin / BS;

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

    // per-warp softmax state (consumers); declared here so the merge can see it
    float o[Gm::kNtO][4];
    float m_lo = -INFINITY, m_hi = -INFINITY, l_lo = 0.f, l_hi = 0.f;
#pragma unroll
    for (int i = 0; i < Gm::kNtO; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;

    if (warp == kConsumerWarps) {
        // ================= producer warp =================
        if (lane == 0) {
            tma_prefetch_desc(&kmap);
            tma_prefetch_desc(&vmap);
        }
        const uint64_t pol = l2_policy_evict_first();
        const int32_t* table = a.block_tables + static_cast<size_t>(s) * a.max_blocks_per_seq + blk0;
        bool ok = true;
        int issued = 0;
        for (int j0 = 0; j0 < nblk && ok; j0 += 32) {
            const int jj = j0 + lane;
            int pid = 0;
            bool bad = false;
            if (jj < nblk) {
                pid = __ldg(table + jj);
                bad = pid < 0 || pid >= a.num_blocks;
            }
            if (__any_sync(0xffffffffu, bad) && lane == 0) {
                raise_error(a.err, PKV_DEVERR_BLOCK_ID);
                *s_abort = 1;
            }
            if (bad) pid = 0;   // load an in-range block; the output becomes NaN
            const int cnt = min(32, nblk - j0);
            for (int i = 0; i < cnt; ++i) {
                const int j = j0 + i;
                const int pj = __shfl_sync(0xffffffffu, pid, i);
                const int stage = j % NST;
                if (lane == 0) {
                    if (j >= NST && !mbar_wait(bar_empty + 8 * stage, ((j / NST) - 1) & 1)) ok = false;
                    if (ok) {
                        const uint32_t fb = bar_full + 8 * stage;
                        const uint32_t kdst = base + stage * Gm::kStageBytes;
                        const uint32_t vdst = kdst + Gm::kTileBytes;
                        mbar_arrive_expect_tx(fb, Gm::kStageBytes);
#pragma unroll
                        for (int sub = 0; sub < Gm::kNsub; ++sub) {
                            tma_load_4d(kdst + sub * Gm::kSubBytes, &kmap, fb, sub * (128 / Gm::E), 0, kvh, pj, pol);
                            tma_load_4d(vdst + sub * Gm::kSubBytes, &vmap, fb, sub * (128 / Gm::E), 0, kvh, pj, pol);
                        }
                        issued = j + 1;
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
        const bool lo_ok = r < G, hi_ok = kHi && (r + 8) < G;
        // Q fragments (A operand, rows = query heads of the group)
        uint32_t qa[Gm::kKsteps][4];
        {
            const uint16_t* qbase = static_cast<const uint16_t*>(a.q) + out_row0 * D;
            const uint32_t* qlo = reinterpret_cast<const uint32_t*>(qbase + static_cast<size_t>(lo_ok ? r : 0) * D);
            const uint32_t* qhi = reinterpret_cast<const uint32_t*>(qbase + static_cast<size_t>(hi_ok ? r + 8 : 0) * D);
#pragma unroll
            for (int ks = 0; ks < Gm::kKsteps; ++ks) {
                const int b2 = Gm::k_base(c, ks) >> 1;
                qa[ks][0] = lo_ok ? __ldg(qlo + b2) : 0u;
                qa[ks][1] = hi_ok ? __ldg(qhi + b2) : 0u;
                qa[ks][2] = lo_ok ? __ldg(qlo + b2 + 1) : 0u;
                qa[ks][3] = hi_ok ? __ldg(qhi + b2 + 1) : 0u;
            }
        }
        const float qk = a.qk_scale_log2;
        for (int j = warp; j < nblk; j += kConsumerWarps) {
            const int stage = j % NST;
            const bool got = mbar_wait(bar_full + 8 * stage, (j / NST) & 1);
            if (!__all_sync(0xffffffffu, got)) {
                if (lane == 0) {
                    raise_error(a.err, PKV_DEVERR_TIMEOUT);
                    *s_abort = 1;
                }
                break;
            }
            const uint32_t kt = base + stage * Gm::kStageBytes;
            const uint32_t vt = kt + Gm::kTileBytes;
            const int valid = min(BS, tok_end - (tok_begin + j * BS));

            // ---- S = Q K^T ----
            float sc[Gm::kNtS][4];
#pragma unroll
            for (int nt = 0; nt < Gm::kNtS; ++nt) {
                sc[nt][0] = sc[nt][1] = sc[nt][2] = sc[nt][3] = 0.f;
                const int row = nt * 8 + r;
                uint4 kw[2 * Gm::kNsub];
#pragma unroll
                for (int qc = 0; qc < 2 * Gm::kNsub; ++qc)
                    kw[qc] = lds128(kt + (qc >> 1) * Gm::kSubBytes + swz128(row, 2 * c + (qc & 1)));
#pragma unroll
                for (int ks = 0; ks < Gm::kKsteps; ++ks) {
                    const uint4& v = kw[ks / Gm::kKpc];
                    uint32_t b0, b1;
                    if constexpr (Gm::E == 2) {
                        const int w0 = (ks % Gm::kKpc) * 2;
                        b0 = word(v, w0);
                        b1 = word(v, w0 + 1);
                    } else {
                        const uint32_t x = word(v, ks % Gm::kKpc);
                        b0 = widen_e4m3x2<kBf16>(x);
                        b1 = widen_e4m3x2<kBf16>(x >> 16);
                    }
                    mma16816<kBf16>(sc[nt], qa[ks], b0, b1);
                }
            }
            // ---- scale, mask, online softmax ----
            float mx_lo = -INFINITY, mx_hi = -INFINITY;
#pragma unroll
            for (int nt = 0; nt < Gm::kNtS; ++nt) {
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int col = nt * 8 + 2 * c + (e & 1);
                    const float x = sc[nt][e] * qk;
                    sc[nt][e] = col < valid ? x : -INFINITY;
                }
                mx_lo = fmaxf(mx_lo, fmaxf(sc[nt][0], sc[nt][1]));
                if constexpr (kHi) mx_hi = fmaxf(mx_hi, fmaxf(sc[nt][2], sc[nt][3]));
            }
            mx_lo = fmaxf(mx_lo, __shfl_xor_sync(0xffffffffu, mx_lo, 1));
            mx_lo = fmaxf(mx_lo, __shfl_xor_sync(0xffffffffu, mx_lo, 2));
            const float mnew_lo = fmaxf(m_lo, mx_lo);
            const float alpha_lo = exp2f(m_lo - mnew_lo);
            m_lo = mnew_lo;
            float alpha_hi = 1.f;
            if constexpr (kHi) {
                mx_hi = fmaxf(mx_hi, __shfl_xor_sync(0xffffffffu, mx_hi, 1));
                mx_hi = fmaxf(mx_hi, __shfl_xor_sync(0xffffffffu, mx_hi, 2));
                const float mnew_hi = fmaxf(m_hi, mx_hi);
                alpha_hi = exp2f(m_hi - mnew_hi);
                m_hi = mnew_hi;
            }
            float sum_lo = 0.f, sum_hi = 0.f;
#pragma unroll
            for (int nt = 0; nt < Gm::kNtS; ++nt) {
                sc[nt][0] = exp2f(sc[nt][0] - m_lo);
                sc[nt][1] = exp2f(sc[nt][1] - m_lo);
                sum_lo += sc[nt][0] + sc[nt][1];
                if constexpr (kHi) {
                    sc[nt][2] = exp2f(sc[nt][2] - m_hi);
                    sc[nt][3] = exp2f(sc[nt][3] - m_hi);
                    sum_hi += sc[nt][2] + sc[nt][3];
                } else {
                    sc[nt][2] = sc[nt][3] = 0.f;
                }
            }
            l_lo = l_lo * alpha_lo + sum_lo;
            if constexpr (kHi) l_hi = l_hi * alpha_hi + sum_hi;
#pragma unroll
            for (int nt = 0; nt < Gm::kNtO; ++nt) {
                o[nt][0] *= alpha_lo;
                o[nt][1] *= alpha_lo;
                if constexpr (kHi) {
                    o[nt][2] *= alpha_hi;
                    o[nt][3] *= alpha_hi;
                }
            }
            // ---- O += P V ----
#pragma unroll
            for (int kk = 0; kk < Gm::kKkPV; ++kk) {
                uint32_t pa[4], pl[4];
                pa[0] = pack2<kBf16>(sc[2 * kk][0], sc[2 * kk][1]);
                pa[1] = pack2<kBf16>(sc[2 * kk][2], sc[2 * kk][3]);
                pa[2] = pack2<kBf16>(sc[2 * kk + 1][0], sc[2 * kk + 1][1]);
                pa[3] = pack2<kBf16>(sc[2 * kk + 1][2], sc[2 * kk + 1][3]);
                if constexpr (kBf16) {
                    pl[0] = pack2<true>(bf16_residual(sc[2 * kk][0]), bf16_residual(sc[2 * kk][1]));
                    pl[1] = pack2<true>(bf16_residual(sc[2 * kk][2]), bf16_residual(sc[2 * kk][3]));
                    pl[2] = pack2<true>(bf16_residual(sc[2 * kk + 1][0]), bf16_residual(sc[2 * kk + 1][1]));
                    pl[3] = pack2<true>(bf16_residual(sc[2 * kk + 1][2]), bf16_residual(sc[2 * kk + 1][3]));
                }
                const int t0 = kk * 16 + 2 * c;     // this thread's four V rows: t0, t0+1, t0+8, t0+9
                constexpr int kVsub = Gm::E == 2 ? Gm::kNsub : 1;
#pragma unroll
                for (int sub = 0; sub < kVsub; ++sub) {
                    const uint32_t vs = vt + sub * Gm::kSubBytes;
                    uint4 v0 = lds128(vs + swz128(t0, r));
                    uint4 v1 = lds128(vs + swz128(t0 + 1, r));
                    uint4 v2 = lds128(vs + swz128(t0 + 8, r));
                    uint4 v3 = lds128(vs + swz128(t0 + 9, r));
                    if (valid < BS) {
                        const uint4 z = make_uint4(0u, 0u, 0u, 0u);
                        if (t0 >= valid) v0 = z;
                        if (t0 + 1 >= valid) v1 = z;
                        if (t0 + 8 >= valid) v2 = z;
                        if (t0 + 9 >= valid) v3 = z;
                    }
#pragma unroll
                    for (int w = 0; w < 4; ++w) {
                        const uint32_t x0 = word(v0, w), x1 = word(v1, w), x2 = word(v2, w), x3 = word(v3, w);
                        if constexpr (Gm::E == 2) {
#pragma unroll
                            for (int h = 0; h < 2; ++h) {
                                const uint32_t sel = h ? 0x7632u : 0x5410u;
                                const uint32_t b0 = __byte_perm(x0, x1, sel);
                                const uint32_t b1 = __byte_perm(x2, x3, sel);
                                const int nt = sub * 8 + 2 * w + h;
                                mma16816<kBf16>(o[nt], pa, b0, b1);
                                if constexpr (kBf16) mma16816<kBf16>(o[nt], pl, b0, b1);
                            }
                        } else {
                            const uint32_t e01 = __byte_perm(x0, x1, 0x5140u), e23 = __byte_perm(x2, x3, 0x5140u);
                            const uint32_t f01 = __byte_perm(x0, x1, 0x7362u), f23 = __byte_perm(x2, x3, 0x7362u);
                            const uint32_t bb[4][2] = {{e01, e23}, {e01 >> 16, e23 >> 16}, {f01, f23}, {f01 >> 16, f23 >> 16}};
#pragma unroll
                            for (int q = 0; q < 4; ++q) {
                                const uint32_t b0 = widen_e4m3x2<kBf16>(bb[q][0]);
                                const uint32_t b1 = widen_e4m3x2<kBf16>(bb[q][1]);
                                const int nt = 4 * w + q;
                                mma16816<kBf16>(o[nt], pa, b0, b1);
                                if constexpr (kBf16) mma16816<kBf16>(o[nt], pl, b0, b1);
                            }
                        }
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_empty + 8 * stage);
        }
        // complete the row sums across the quad
        l_lo += __shfl_xor_sync(0xffffffffu, l_lo, 1);
        l_lo += __shfl_xor_sync(0xffffffffu, l_lo, 2);
        if constexpr (kHi) {
            l_hi += __shfl_xor_sync(0xffffffffu, l_hi, 1);
            l_hi += __shfl_xor_sync(0xffffffffu, l_hi, 2);
        }
    }
    __syncthreads();   // ring fully consumed: reuse it for the merge

    float* sm_o = reinterpret_cast<float*>(gbase);                    // [warps][16][D]
    float* sm_m = sm_o + kConsumerWarps * 16 * D;                      // [warps][16]
    float* sm_l = sm_m + kConsumerWarps * 16;                          // [warps][16]
    if (warp < kConsumerWarps) {
        const int r = lane >> 2, c = lane & 3;
        float* ow = sm_o + warp * 16 * D;
#pragma unroll
        for (int nt = 0; nt < Gm::kNtO; ++nt) {
            const int d0 = Gm::o_dim(nt, 2 * c), d1 = Gm::o_dim(nt, 2 * c + 1);
            ow[r * D + d0] = o[nt][0];
            ow[r * D + d1] = o[nt][1];
            if constexpr (kHi) {
                ow[(r + 8) * D + d0] = o[nt][2];
                ow[(r + 8) * D + d1] = o[nt][3];
            }
        }
        if (c == 0) {
            sm_m[warp * 16 + r] = m_lo;
            sm_l[warp * 16 + r] = l_lo;
            if constexpr (kHi) {
                sm_m[warp * 16 + r + 8] = m_hi;
                sm_l[warp * 16 + r + 8] = l_hi;
            }
        }
    }
    __syncthreads();
    const bool aborted = *s_abort != 0;
    const bool single = nparts == 1;
    for (int e = threadIdx.x; e < G * D; e += kThreads) {
        const int hh = e / D, d = e - hh * D;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kConsumerWarps; ++w) M = fmaxf(M, sm_m[w * 16 + hh]);
        float num = 0.f, den = 0.f;
#pragma unroll
        for (int w = 0; w < kConsumerWarps; ++w) {
            const float f = exp2f(sm_m[w * 16 + hh] - M);
            num += f * sm_o[(w * 16 + hh) * D + d];
            den += f * sm_l[w * 16 + hh];
        }
        float val = num / den * a.v_scale;
        if (aborted) val = __int_as_float(0x7fc00000);
        if (single) {
            store_out<kQBf16>(a.out, (out_row0 + hh) * D + d, val);
        } else {
            const size_t slot = (out_row0 + hh) * a.max_partitions + part;
            a.ws_o[slot * D + d] = val;
            if (d == 0) a.ws_ml[slot] = make_float2(aborted ? __int_as_float(0x7fc00000) : M, den);
        }
    }
}

// ---- pass 2: merge partitions by log-sum-exp -------------------------------------

template <bool kQBf16, int D>
__global__ void __launch_bounds__(D) decode_reduce_kernel(const DecodeArgs a) {
    const int qh = blockIdx.x, s = blockIdx.y, d = threadIdx.x;
    const int L = __ldg(a.context_lens + s);
    if (L <= 0 || L > a.max_blocks_per_seq * a.block_size || L > a.max_context_len) return;
    const int nparts = (L + a.partition_size - 1) / a.partition_size;
    if (nparts <= 1) return;
    const size_t row = static_cast<size_t>(s) * a.num_heads + qh;
    const float2* ml = a.ws_ml + row * a.max_partitions;
    const float* wo = a.ws_o + row * a.max_partitions * D;
    float M = -INFINITY;
    for (int p = 0; p < nparts; ++p) M = fmaxf(M, ml[p].x);
    float num = 0.f, den = 0.f;
    for (int p = 0; p < nparts; ++p) {
        const float2 v = ml[p];
        const float w = exp2f(v.x - M) * v.y;
        num += w * wo[static_cast<size_t>(p) * D + d];
        den += w;
    }
    store_out<kQBf16>(a.out, row * D + d, num / den);
}

// ---- host side -----------------------------------------------------------------------

int pick_partition(int num_seqs, int num_kv_heads, int block_size, int max_context_len, int requested) {
    const int cap = ((max_context_len > 0 ? max_context_len : 1) + block_size - 1) / block_size * block_size;
    if (requested > 0) return requested >= cap ? cap : requested;
    int p = 512 < cap ? 512 : cap;
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
pkv_status launch_decode(const DecodeArgs& a, const CUtensorMap& km, const CUtensorMap& vm,
                         cudaStream_t st) {
    using Gm = Geo<KV, D, BS>;
    auto kern = paged_decode_kernel<KV, kQBf16, D, BS, kHi>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Gm::kSmemBytes) != cudaSuccess)
        return PKV_ERR_CUDA;
    dim3 grid(a.max_partitions, a.num_kv_heads, a.num_seqs);
    kern<<<grid, kThreads, Gm::kSmemBytes, st>>>(a, km, vm);
    if (cudaGetLastError() != cudaSuccess) return PKV_ERR_CUDA;
    if (a.max_partitions > 1) {
        decode_reduce_kernel<kQBf16, D><<<dim3(a.num_heads, a.num_seqs), D, 0, st>>>(a);
        if (cudaGetLastError() != cudaSuccess) return PKV_ERR_CUDA;
    }
    return PKV_OK;
}

template <int KV, bool kQBf16, int D>
pkv_status dispatch_bs(const DecodeArgs& a, const CUtensorMap& km, const CUtensorMap& vm, cudaStream_t st,
                       bool hi) {
    if (a.block_size == 16)
        return hi ? launch_decode<KV, kQBf16, D, 16, true>(a, km, vm, st)
                  : launch_decode<KV, kQBf16, D, 16, false>(a, km, vm, st);
    return hi ? launch_decode<KV, kQBf16, D, 32, true>(a, km, vm, st)
              : launch_decode<KV, kQBf16, D, 32, false>(a, km, vm, st);
}

}  // namespace
}  // namespace pkv

extern "C" int pkv_decode_partition_size(int num_seqs, int num_kv_heads, int block_size, int max_context_len,
                                         int partition_size) {
    if (num_seqs < 0 || num_kv_heads <= 0 || block_size <= 0 || max_context_len < 0 || partition_size < 0 ||
        partition_size % block_size != 0)
        return 0;
    return pkv::pick_partition(num_seqs, num_kv_heads, block_size, max_context_len, partition_size);
}

extern "C" size_t pkv_decode_workspace_bytes(int num_seqs, int num_heads, int num_kv_heads, int head_dim,
                                             int block_size, int max_context_len, int partition_size) {
    const int ps = pkv_decode_partition_size(num_seqs, num_kv_heads, block_size, max_context_len, partition_size);
    if (ps <= 0 || num_heads <= 0 || head_dim <= 0) return 0;
    const long long parts = (static_cast<long long>(max_context_len) + ps - 1) / ps;
    if (parts <= 1) return 0;
    const size_t rows = static_cast<size_t>(num_seqs) * num_heads * static_cast<size_t>(parts);
    const size_t o_bytes = (rows * head_dim * sizeof(float) + 255) / 256 * 256;
    return o_bytes + rows * sizeof(float2);
}

extern "C" pkv_status pkv_paged_attn_decode(void* out, const void* q, pkv_dtype q_dtype, const void* k_pool,
                                            const void* v_pool, pkv_dtype kv_dtype, float k_scale, float v_scale,
                                            const int32_t* block_tables, int max_blocks_per_seq,
                                            const int32_t* context_lens, int max_context_len, int num_seqs,
                                            int num_heads, int num_kv_heads, int head_dim, int block_size,
                                            int num_blocks, float scale, int partition_size, void* workspace,
                                            size_t workspace_bytes, uint32_t* device_error, void* stream) {
    using namespace pkv;
    if (num_seqs < 0 || num_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 ||
        num_blocks <= 0 || max_blocks_per_seq <= 0 || max_context_len < 0 || partition_size < 0)
        return PKV_ERR_INVALID_ARG;
    if (num_heads % num_kv_heads != 0) return PKV_ERR_INVALID_ARG;
    if (!(scale == scale)) return PKV_ERR_INVALID_ARG;
    const int G = num_heads / num_kv_heads;
    if (G > 16) return PKV_ERR_UNSUPPORTED;
    if (block_size != 16 && block_size != 32) return PKV_ERR_UNSUPPORTED;
    if (partition_size % block_size != 0) return PKV_ERR_INVALID_ARG;
    if (q_dtype != PKV_F16 && q_dtype != PKV_BF16) return PKV_ERR_UNSUPPORTED;
    if (kv_dtype != q_dtype && kv_dtype != PKV_FP8_E4M3) return PKV_ERR_UNSUPPORTED;
    if (kv_dtype == PKV_FP8_E4M3) {
        if (head_dim != 128) return PKV_ERR_UNSUPPORTED;
        if (!(k_scale > 0.f && v_scale > 0.f)) return PKV_ERR_INVALID_ARG;
    } else if (head_dim != 64 && head_dim != 128) {
        return PKV_ERR_UNSUPPORTED;
    }
    if (num_seqs > 65535 || num_kv_heads > 65535) return PKV_ERR_UNSUPPORTED;
    if (num_seqs == 0) return PKV_OK;
    if (!out || !q || !k_pool || !v_pool || !block_tables || !context_lens) return PKV_ERR_INVALID_ARG;
    if (!aligned16(out) || !aligned16(q) || !aligned16(k_pool) || !aligned16(v_pool) ||
        (reinterpret_cast<uintptr_t>(block_tables) & 3) || (reinterpret_cast<uintptr_t>(context_lens) & 3))
        return PKV_ERR_ALIGNMENT;

    const int ps = pick_partition(num_seqs, num_kv_heads, block_size, max_context_len, partition_size);
    const int parts = max_context_len > 0 ? (max_context_len + ps - 1) / ps : 1;
    const size_t need = pkv_decode_workspace_bytes(num_seqs, num_heads, num_kv_heads, head_dim, block_size,
                                                   max_context_len, partition_size);
    if (need > 0 && (!workspace || workspace_bytes < need)) return PKV_ERR_WORKSPACE;
    if (need > 0 && (reinterpret_cast<uintptr_t>(workspace) & 255)) return PKV_ERR_ALIGNMENT;

    DecodeArgs a{};
    a.out = out;
    a.q = q;
    a.block_tables = block_tables;
    a.context_lens = context_lens;
    const size_t rows = static_cast<size_t>(num_seqs) * num_heads * static_cast<size_t>(parts);
    a.ws_o = need ? static_cast<float*>(workspace) : nullptr;
    a.ws_ml = need ? reinterpret_cast<float2*>(static_cast<uint8_t*>(workspace) +
                                               (rows * head_dim * sizeof(float) + 255) / 256 * 256)
                   : nullptr;
    a.err = device_error;
    a.max_blocks_per_seq = max_blocks_per_seq;
    a.max_context_len = max_context_len;
    a.num_seqs = num_seqs;
    a.num_heads = num_heads;
    a.num_kv_heads = num_kv_heads;
    a.num_blocks = num_blocks;
    a.block_size = block_size;
    a.partition_size = ps;
    a.max_partitions = parts;
    const float ks = kv_dtype == PKV_FP8_E4M3 ? k_scale : 1.f;
    a.qk_scale_log2 = static_cast<float>(static_cast<double>(scale) * ks * 1.4426950408889634);
    a.v_scale = kv_dtype == PKV_FP8_E4M3 ? v_scale : 1.f;

    alignas(64) CUtensorMap km;
    alignas(64) CUtensorMap vm;
    if (!encode_pool_map(&km, k_pool, kv_dtype, head_dim, block_size, num_kv_heads, num_blocks) ||
        !encode_pool_map(&vm, v_pool, kv_dtype, head_dim, block_size, num_kv_heads, num_blocks))
        return PKV_ERR_CUDA;

    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const bool hi = G > 8;
    const bool qbf = q_dtype == PKV_BF16;
    switch (kv_dtype) {
    case PKV_F16:
        return head_dim == 64 ? dispatch_bs<KV_F16, false, 64>(a, km, vm, st, hi)
                              : dispatch_bs<KV_F16, false, 128>(a, km, vm, st, hi);
    case PKV_BF16:
        return head_dim == 64 ? dispatch_bs<KV_BF16, true, 64>(a, km, vm, st, hi)
                              : dispatch_bs<KV_BF16, true, 128>(a, km, vm, st, hi);
    case PKV_FP8_E4M3:
        return qbf ? dispatch_bs<KV_E4M3, true, 128>(a, km, vm, st, hi)
                   : dispatch_bs<KV_E4M3, false, 128>(a, km, vm, st, hi);
    }
    return PKV_ERR_UNSUPPORTED;
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
// that device; make that first call before any stream capture.

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
    const size_t need = pkv_decode_workspace_bytes(num_seqs, num_heads, num_kv_heads, head_dim, block_size,
                                                   max_context_len, partition_size);
    if (need > pkv::kStaticWsBytes) return PKV_ERR_WORKSPACE;
    void* ws = nullptr;
    if (need > 0 && pkv::static_ws_address(&ws) != cudaSuccess) return PKV_ERR_CUDA;
    return pkv_paged_attn_decode(out, q, q_dtype, k_pool, v_pool, kv_dtype, k_scale, v_scale, block_tables,
                                 max_blocks_per_seq, context_lens, max_context_len, num_seqs, num_heads,
                                 num_kv_heads, head_dim, block_size, num_blocks, scale, partition_size, ws,
                                 need > 0 ? pkv::kStaticWsBytes : 0, device_error, stream);
}
