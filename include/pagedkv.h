/*
 * pagedkv.h -- C ABI of the B200 (sm_100a) paged KV-cache library.
 *
 * The KV cache of every sequence is split into fixed-size blocks that sit
 * anywhere in one shared physical pool and are reached through a
 * per-sequence block table (Ultralytics glossary "PagedAttention", section
 * "How paging works"; Wikipedia "PagedAttention", section "Description").
 * The library provides the three GPU operations of a decode step:
 *
 *   pkv_reshape_and_cache  write the new tokens' K/V into the pool through a
 *                          slot mapping (the glossary's worked example:
 *                          pool[table[pos / B], pos % B] = key);
 *   pkv_copy_blocks        block-granular copy-on-write of shared blocks
 *                          (glossary, section "Sharing blocks across
 *                          sequences"; "vLLM and PagedAttention" transcript:
 *                          the partially filled shared block is copied);
 *   pkv_paged_attn_decode  single-query causal attention over the paged pool
 *                          (Wikipedia "PagedAttention", section "Mathematical
 *                          formulation": o_i = sum_j V_j A_ij^T over the
 *                          ceil(i/B) blocks of the sequence).
 * and the prefill of a chunk of new tokens over the same cache
 * (pkv_paged_attn_prefill: every query of the chunk attends causally, the
 * dense phase of the "vLLM and PagedAttention" transcript's opening
 * paragraph), on the 5th-generation tensor cores, also over an E4M3 cache
 * (pkv_paged_attn_prefill_fp8).  Around them: a decode that reads shared
 * prompt blocks once per group of sequences
 * (pkv_paged_attn_decode_shared_prefix), block swapping between the device
 * pool and pinned host memory (pkv_swap_blocks), a host-side block manager
 * with copy-on-write, chunk appends, prefix caching by block content and
 * swap bookkeeping (pkv_bm_*), a host check of copy and swap pair lists
 * (pkv_check_block_pairs), and a read-only pass over a device buffer that
 * measurements quote decode against (pkv_stream_read).
 *
 * Conventions shared by every entry point
 *   - All pointers except scalars are DEVICE pointers, owned by the caller
 *     (exceptions, stated where they apply: the block manager's arrays are
 *     host memory; pkv_swap_blocks also takes pinned, mapped host pools).
 *     The GPU calls allocate nothing (the one exception,
 *     pkv_paged_attn_decode_static_ws, uses a file-scope device array of
 *     the library) and keep no state between calls; calls are
 *     asynchronous on `stream` (a cudaStream_t passed as void*, NULL = the
 *     legacy default stream) and nothing synchronises.
 *   - Pools have layout [num_blocks][num_kv_heads][block_size][head_dim],
 *     row-major, element type kv_dtype.  One (block, kv head) tile is one
 *     contiguous run of block_size * head_dim elements.  K and V pools have
 *     the same layout.  Pool base pointers must be 16-byte aligned.
 *   - A "slot" is block_id * block_size + offset_in_block.
 *   - Problems the host can see (null pointers, unsupported sizes or dtype
 *     pairs, misaligned pointers, an undersized workspace) return a non-zero
 *     status synchronously and launch nothing.  Launch failures return
 *     PKV_ERR_CUDA.  Data-dependent problems are found on the device: the
 *     offending item is skipped (attention writes NaN for the affected
 *     sequence and head group) and a bit is OR-ed into *device_error (if
 *     device_error is not NULL).  Kernels never trap; every wait inside a
 *     kernel is bounded, and a wait that gives up sets PKV_DEVERR_TIMEOUT.
 *     The caller reads *device_error after synchronising and clears it.
 */
#ifndef PAGEDKV_H
#define PAGEDKV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    PKV_OK = 0,
    PKV_ERR_INVALID_ARG = 1,   /* null pointer, negative size, inconsistent sizes */
    PKV_ERR_UNSUPPORTED = 2,   /* valid but not implemented: head_dim, block_size, dtype pair, group size */
    PKV_ERR_WORKSPACE = 3,     /* workspace missing or smaller than pkv_decode_workspace_bytes() */
    PKV_ERR_CUDA = 4,          /* a CUDA runtime or driver call failed */
    PKV_ERR_ALIGNMENT = 5,     /* a pointer is not 16-byte aligned */
    PKV_ERR_OUT_OF_BLOCKS = 6  /* the block manager's free list cannot serve the request */
} pkv_status;

typedef enum {
    PKV_F16 = 0,               /* IEEE binary16 */
    PKV_BF16 = 1,              /* bfloat16 */
    PKV_FP8_E4M3 = 2           /* OCP E4M3 (no infinities, max finite 448), with a per-tensor scale */
} pkv_dtype;

/* Bits OR-ed into *device_error. */
#define PKV_DEVERR_BLOCK_ID    0x1u   /* a block-table entry read by attention is outside [0, num_blocks) */
#define PKV_DEVERR_SLOT        0x2u   /* a slot >= num_blocks * block_size */
#define PKV_DEVERR_PAIR        0x4u   /* a copy pair names a block outside [0, num_blocks) */
#define PKV_DEVERR_CONTEXT_LEN 0x8u   /* context_len < 0, > max_blocks_per_seq * block_size, or > max_context_len */
#define PKV_DEVERR_TIMEOUT     0x10u  /* a bounded wait inside a kernel gave up */

/* Library version: major * 10000 + minor * 100 + patch. */
int pkv_version(void);

/* Human-readable text for a status code (static storage). */
const char* pkv_status_string(pkv_status status);

/*
 * Workspace that pkv_paged_attn_decode needs for the split-context pass
 * (per sequence, query head and partition: running max, sum and a head_dim
 * output vector in float32).  Zero when every sequence fits one partition.
 * partition_size as for pkv_paged_attn_decode (0 = automatic).  Returns 0
 * for invalid arguments as well.
 */
size_t pkv_decode_workspace_bytes(int num_seqs, int num_heads, int num_kv_heads, int head_dim,
                                  pkv_dtype kv_dtype, int block_size, int max_context_len,
                                  int partition_size);

/* The partition size (tokens) that pkv_paged_attn_decode uses for these
 * arguments; equals max_context_len rounded up to block_size when no split
 * happens.  The automatic choice (partition_size 0) aims at about 512 KB of
 * K+V per partition and KV head (1,024 tokens of 16-bit head_dim 128, 2,048 of
 * FP8), shrunk while there are fewer than two work units per SM.  Returns 0
 * for invalid arguments. */
int pkv_decode_partition_size(int num_seqs, int num_kv_heads, int head_dim, pkv_dtype kv_dtype,
                              int block_size, int max_context_len, int partition_size);

/*
 * Paged decode attention (Wikipedia "PagedAttention", section "Mathematical
 * formulation"; FlashAttention-style tiling and GQA as in the glossary's
 * section "Related methods").
 *
 * For each sequence s with L = context_lens[s] (the new token included, so
 * its K/V must already be in the pool) and each query head h:
 *   out[s][h][:] = sum_{t < L} softmax_t(scale * q[s][h] . k_t) * v_t,
 *   k_t = K_pool[block_tables[s][t / block_size]][h / G][t % block_size][:],
 *   G = num_heads / num_kv_heads (contiguous query-head groups share a KV head).
 * For FP8 pools the stored values are multiplied by k_scale / v_scale.
 * L = 0 gives a zero output.  Table entries at j >= ceil(L / block_size) are
 * never read.  Physical blocks may be shared between and within sequences.
 *
 *   out            [num_seqs][num_heads][head_dim], q_dtype
 *   q              [num_seqs][num_heads][head_dim], q_dtype in {F16, BF16}
 *   k_pool/v_pool  see conventions; kv_dtype == q_dtype, or FP8_E4M3
 *   block_tables   int32 [num_seqs][max_blocks_per_seq]
 *   context_lens   int32 [num_seqs]
 *   max_context_len  an upper bound of context_lens (sizes the grid)
 *   head_dim in {64, 128} (128 only for FP8); block_size in {16, 32};
 *   num_heads % num_kv_heads == 0 and G <= 16
 *   partition_size 0 = automatic, else a multiple of block_size: sequences
 *                  longer than it are split into partitions that run in
 *                  parallel and are merged exactly by log-sum-exp
 *   workspace      device buffer of at least pkv_decode_workspace_bytes()
 *                  bytes (may be NULL when that is 0), 256-byte aligned
 *   scale          finite; k_scale, v_scale (FP8 pools only) positive and finite
 */
pkv_status pkv_paged_attn_decode(void* out, const void* q, pkv_dtype q_dtype,
                                 const void* k_pool, const void* v_pool, pkv_dtype kv_dtype,
                                 float k_scale, float v_scale,
                                 const int32_t* block_tables, int max_blocks_per_seq,
                                 const int32_t* context_lens, int max_context_len,
                                 int num_seqs, int num_heads, int num_kv_heads, int head_dim,
                                 int block_size, int num_blocks, float scale, int partition_size,
                                 void* workspace, size_t workspace_bytes,
                                 uint32_t* device_error, void* stream);

/*
 * Shared-prefix decode: pkv_paged_attn_decode's result, computed with each shared
 * prefix read once per unit instead of once per sequence (several sequences whose
 * tables begin with the same full blocks -- parallel samples or beam candidates of
 * one prompt, glossary "PagedAttention", section "Sharing blocks across
 * sequences").  Pass 1 runs every unit's query rows (all heads of up to
 * unit_width members, unit_width * G <= 16) over the unit's shared tokens; pass 2
 * runs every sequence over its own tokens, from the end of its prefix; a merge
 * combines both sets of partials exactly by log-sum-exp.  The prefix pass picks its
 * own partition size (the automatic rule applied to units instead of sequences).
 *
 *   seq_prefix_len  device int32 [num_seqs]: shared tokens of each sequence (a
 *                   multiple of block_size, <= its context length; 0 = none)
 *   unit_seqs       device int32 [num_units][unit_width]: member sequences of each
 *                   unit (-1 pads the last slots); members must share their first
 *                   unit_len[u] / block_size table entries and have that prefix length
 *   unit_len        device int32 [num_units]
 *   max_prefix_len  bound of every seq_prefix_len and unit_len
 *   plan            PKV_PREFIX_PLAN_AUTO: the passes above only when the units'
 *                   shared prefixes, counted once per unit, exceed the device's
 *                   L2 (otherwise the plain call's repeated reads of them hit L2
 *                   and its single pass is faster, so it runs instead);
 *                   PKV_PREFIX_PLAN_SHARED: always the passes above;
 *                   PKV_PREFIX_PLAN_PLAIN: always the plain call
 *   workspace       >= pkv_shared_prefix_workspace_bytes() bytes (always needed)
 * Preconditions, checked on the device: every sequence with seq_prefix_len > 0
 * is a member of exactly one unit, and every member's seq_prefix_len equals its
 * unit's unit_len; members are packed before the -1 pads; no length exceeds
 * max_prefix_len.  A sequence whose prefix no unit covers, every member of a
 * unit that breaks these rules, and a length beyond max_prefix_len get NaN
 * outputs and PKV_DEVERR_CONTEXT_LEN (nothing is read outside the workspace).
 * Other arguments, errors and results as for pkv_paged_attn_decode.
 * pkv_find_shared_prefixes() builds the three arrays from host copies of the tables.
 */
typedef enum {
    PKV_PREFIX_PLAN_AUTO = 0,
    PKV_PREFIX_PLAN_SHARED = 1,
    PKV_PREFIX_PLAN_PLAIN = 2
} pkv_prefix_plan;

/* The plan pkv_paged_attn_decode_shared_prefix carries out for these arguments:
 * PKV_PREFIX_PLAN_SHARED (three launches: tail pass, prefix pass, merge) or
 * PKV_PREFIX_PLAN_PLAIN (pkv_paged_attn_decode's one or two); -1 for an unknown
 * plan.  Reads the current device's L2 size for PKV_PREFIX_PLAN_AUTO. */
int pkv_shared_prefix_plan_used(int num_units, int num_kv_heads, int head_dim, pkv_dtype kv_dtype,
                                int max_prefix_len, int plan);

size_t pkv_shared_prefix_workspace_bytes(int num_seqs, int num_heads, int num_kv_heads, int head_dim,
                                         pkv_dtype kv_dtype, int block_size, int max_context_len,
                                         int num_units, int max_prefix_len, int partition_size);

pkv_status pkv_paged_attn_decode_shared_prefix(void* out, const void* q, pkv_dtype q_dtype,
                                               const void* k_pool, const void* v_pool, pkv_dtype kv_dtype,
                                               float k_scale, float v_scale,
                                               const int32_t* block_tables, int max_blocks_per_seq,
                                               const int32_t* context_lens, int max_context_len,
                                               int num_seqs, int num_heads, int num_kv_heads, int head_dim,
                                               int block_size, int num_blocks, float scale, int partition_size,
                                               const int32_t* seq_prefix_len, const int32_t* unit_seqs,
                                               const int32_t* unit_len, int num_units, int unit_width,
                                               int max_prefix_len, int plan, void* workspace,
                                               size_t workspace_bytes,
                                               uint32_t* device_error, void* stream);

/*
 * Host helper (HOST arrays): groups sequences whose tables start with the same
 * block ids, takes the longest run of leading blocks common to a group and full in
 * every member as its shared prefix, and packs each group into units of at most
 * unit_width members.  Sequences alone in their group get prefix 0 and no unit.
 * Fills seq_prefix_len [num_seqs], unit_seqs [max_units][unit_width], unit_len
 * [max_units], *num_units and *max_prefix_len; PKV_ERR_INVALID_ARG if more than
 * max_units units are needed.
 */
pkv_status pkv_find_shared_prefixes(const int32_t* block_tables, const int32_t* context_lens, int num_seqs,
                                    int max_blocks_per_seq, int block_size, int unit_width,
                                    int32_t* seq_prefix_len, int32_t* unit_seqs, int32_t* unit_len,
                                    int max_units, int* num_units, int* max_prefix_len);

/*
 * Size of the library-owned workspace used by pkv_paged_attn_decode_static_ws
 * (64 MiB of device memory, held by every GPU that loads the library).
 */
#define PKV_STATIC_WORKSPACE_BYTES (64ull << 20)

/*
 * pkv_paged_attn_decode for callers that cannot allocate device memory.  The
 * pages describe no such call; it exists for this library's users: code that
 * runs inside a host framework owning every device allocation, or a serving
 * loop that must not allocate once running (cudaMalloc may synchronise the
 * device).  The caller still passes inputs and outputs; the split-context
 * workspace is a file-scope device array of PKV_STATIC_WORKSPACE_BYTES inside
 * the library, so this call allocates nothing.
 *
 * Arguments and results are those of pkv_paged_attn_decode, minus workspace.
 * Returns PKV_ERR_WORKSPACE, launching nothing, when the call would need more
 * than PKV_STATIC_WORKSPACE_BYTES (pkv_decode_workspace_bytes tells).  The
 * first call on each device looks up the array's device address (with that
 * device current); make that first call before any stream capture.  Every
 * call shares the one array and leaves its contents behind (nothing in it
 * needs to start at zero: each call writes every entry it reads), so calls
 * that overlap on the GPU -- concurrent streams, or several host threads --
 * race on it; serialise them.  Arguments are checked exactly as for
 * pkv_paged_attn_decode before the size test.  The looked-up address is kept
 * for the life of the process and does not survive cudaDeviceReset: do not
 * use this call after one.
 */
pkv_status pkv_paged_attn_decode_static_ws(void* out, const void* q, pkv_dtype q_dtype,
                                           const void* k_pool, const void* v_pool, pkv_dtype kv_dtype,
                                           float k_scale, float v_scale,
                                           const int32_t* block_tables, int max_blocks_per_seq,
                                           const int32_t* context_lens, int max_context_len,
                                           int num_seqs, int num_heads, int num_kv_heads, int head_dim,
                                           int block_size, int num_blocks, float scale, int partition_size,
                                           uint32_t* device_error, void* stream);

/*
 * Chunked prefill over the paged cache (Wikipedia "PagedAttention", section
 * "Mathematical formulation", token form, for every query position of a
 * chunk; "vLLM and PagedAttention" transcript, opening paragraph: the prompt
 * is processed at once as large matrix products; "Paged Attention" study
 * notes (huajishe.fun), section on points to watch: prefill needs its own
 * handling).
 *
 * Sequence s holds L = context_lens[s] tokens in the pool, the last
 * C = query_start[s+1] - query_start[s] of which are the chunk (their K/V
 * already written, e.g. by pkv_reshape_and_cache).  Query row
 * r = query_start[s] + j (0 <= j < C) sits at position p = L - C + j:
 *   out[r][h][:] = sum_{t <= p} softmax_t(scale * q[r][h] . k_t) * v_t,
 * with k_t, v_t read through the block table as in decode and
 * h / G the KV head of query head h.  Decode is the case C = 1.
 *
 *   out            [num_tokens][num_heads][head_dim], dtype
 *   q              [num_tokens][num_heads][head_dim], dtype in {F16, BF16};
 *                  the chunks of all sequences packed in order
 *   k_pool/v_pool  see conventions, the same dtype as q
 *   block_tables   int32 [num_seqs][max_blocks_per_seq]
 *   context_lens   int32 [num_seqs]
 *   query_start    int32 [num_seqs + 1], query_start[0] = 0,
 *                  query_start[num_seqs] = num_tokens, non-decreasing
 *   max_query_len  an upper bound of the chunk lengths (sizes the grid)
 *   head_dim in {64, 128}; block_size in {16, 32}; G = num_heads /
 *   num_kv_heads in {1, 2, 4, 8, 16}; scale > 0.
 *   workspace      BF16 only, optional (see below): device memory of at least
 *                  pkv_prefill_workspace_bytes() bytes, 256-byte aligned, or
 *                  null; ignored for F16.  Owned by the caller, unused after
 *                  the call's kernels complete.
 * Data-dependent problems (a chunk longer than its context, a context beyond
 * the table, a bad block id) write NaN rows for the affected query tile and
 * set PKV_DEVERR_CONTEXT_LEN / PKV_DEVERR_BLOCK_ID.  Scores and the output
 * accumulate in float32.  The softmax weights P enter the P.V tensor-core
 * product as f16 (11 significant bits).  A bf16 V cannot meet an f16 P in
 * one product, so for BF16:
 *   - with a workspace, two passes first narrow V to f16 in the workspace:
 *     for each (sequence, KV head) the power of two 2^e that brings its
 *     largest finite |v| (positions < context_len) into [2^15, 2^16), then
 *     v * 2^-e rounded to f16 (exact down to 2^-29 of that maximum; Inf and
 *     NaN kept), and 2^e multiplies the head's output rows;
 *   - without one, P enters as a bf16 high part plus a bf16 low part
 *     (P - bf16(P)) against the bf16 V: two products, slower, no memory.
 * For BF16, returns PKV_ERR_WORKSPACE if a non-null workspace is smaller
 * than pkv_prefill_workspace_bytes() and PKV_ERR_ALIGNMENT if it is not
 * 256-byte aligned, launching nothing.  pkv_prefill_workspace_bytes() is 0
 * for F16 (and any dtype but BF16) and for non-positive sizes.
 */
size_t pkv_prefill_workspace_bytes(pkv_dtype dtype, int num_seqs, int max_blocks_per_seq, int num_kv_heads,
                                   int head_dim, int block_size);
pkv_status pkv_paged_attn_prefill(void* out, const void* q, pkv_dtype dtype, const void* k_pool,
                                  const void* v_pool, const int32_t* block_tables, int max_blocks_per_seq,
                                  const int32_t* context_lens, const int32_t* query_start, int max_query_len,
                                  int num_seqs, int num_tokens, int num_heads, int num_kv_heads, int head_dim,
                                  int block_size, int num_blocks, float scale, void* workspace,
                                  size_t workspace_bytes, uint32_t* device_error, void* stream);

/*
 * Chunked prefill over an FP8_E4M3 cache (glossary, section "Related methods":
 * an 8-bit KV cache), same result definition as pkv_paged_attn_prefill with
 * k_t = e4m3(K byte) * k_scale and v_t = e4m3(V byte) * v_scale.  A gather
 * kernel widens the blocks each sequence's queries can reach into 16-bit
 * pools inside `workspace` (one row of max_blocks_per_seq blocks per
 * sequence; both exactly: K to q_dtype, V to f16), then the tensor-core
 * prefill runs on them with scale * k_scale, one f16 P.V product, and
 * v_scale multiplying the output rows.  Arguments as for
 * pkv_paged_attn_prefill, except: q_dtype in {F16, BF16} is also the output
 * type; the pools hold E4M3 bytes; k_scale, v_scale > 0; workspace: device
 * memory of at least pkv_prefill_fp8_workspace_bytes() bytes, 256-byte
 * aligned.  A bad block id yields PKV_DEVERR_BLOCK_ID and NaN rows.
 */
size_t pkv_prefill_fp8_workspace_bytes(int num_seqs, int max_blocks_per_seq, int num_kv_heads, int head_dim,
                                       int block_size);
pkv_status pkv_paged_attn_prefill_fp8(void* out, const void* q, pkv_dtype q_dtype, const void* k_pool,
                                      const void* v_pool, float k_scale, float v_scale, const int32_t* block_tables,
                                      int max_blocks_per_seq, const int32_t* context_lens,
                                      const int32_t* query_start, int max_query_len, int num_seqs, int num_tokens,
                                      int num_heads, int num_kv_heads, int head_dim, int block_size, int num_blocks,
                                      float scale, void* workspace, size_t workspace_bytes, uint32_t* device_error,
                                      void* stream);

/*
 * Scatter new tokens into the pool (glossary "PagedAttention", section "How
 * paging works").  For every token t with slot = slot_mapping[t] >= 0 and
 * every KV head h:
 *   k_pool[slot / block_size][h][slot % block_size][:] = k[t][h][:]  (same for v)
 * copied bit for bit when kv_dtype == in_dtype; for an FP8_E4M3 pool each
 * element is stored as e4m3(x / scale), the division in IEEE float32 and the
 * conversion round-to-nearest-even saturating at +-448.  Negative slots are
 * skipped.  Slots must be distinct (two tokens writing one slot race).
 *
 *   k, v           [num_tokens][num_kv_heads][head_dim], in_dtype in {F16, BF16}, 16-byte aligned
 *   slot_mapping   int64 [num_tokens]
 *   head_dim       a multiple of 8
 *   k_scale, v_scale   E4M3 pools only: positive and finite (else PKV_ERR_INVALID_ARG)
 */
pkv_status pkv_reshape_and_cache(const void* k, const void* v, pkv_dtype in_dtype,
                                 void* k_pool, void* v_pool, pkv_dtype kv_dtype,
                                 float k_scale, float v_scale,
                                 const int64_t* slot_mapping, int num_tokens,
                                 int num_kv_heads, int head_dim, int block_size, int num_blocks,
                                 uint32_t* device_error, void* stream);

/*
 * Block-granular copy-on-write (glossary "PagedAttention", section "Sharing
 * blocks across sequences"): for every pair i,
 *   k_pool[pairs[i][1]] := k_pool[pairs[i][0]] and the same for v_pool,
 * block_bytes = num_kv_heads * block_size * head_dim * element size, a
 * multiple of 16.  pairs is int64 [num_pairs][2] (src, dst) in device memory.
 * Precondition (not checked on the device; pkv_check_block_pairs checks a
 * host copy): destinations are distinct and no destination is also a source,
 * so the copies are independent.
 */
pkv_status pkv_copy_blocks(void* k_pool, void* v_pool, size_t block_bytes,
                           const int64_t* pairs, int num_pairs, int num_blocks,
                           uint32_t* device_error, void* stream);

/*
 * Block swap between two pools of the same layout ("vLLM and PagedAttention"
 * transcript, on preemption: a group's KV data moves to CPU memory and comes
 * back later): for every pair i,
 *   dst_k_pool[pairs[i][1]] := src_k_pool[pairs[i][0]] and the same for V,
 * block_bytes = num_kv_heads * block_size * head_dim * element size, a
 * multiple of 16.  Each pool is device memory or host memory pinned and
 * mapped by CUDA (cudaHostAlloc, or torch's pin_memory) -- the kernel reads or
 * writes it across the link directly; pageable host memory is rejected with
 * PKV_ERR_INVALID_ARG.  pairs is int64 [num_pairs][2] (src block, dst block),
 * device or mapped host memory; pkv_bm_swap produces it.  Pairs naming a
 * block outside [0, src_num_blocks) / [0, dst_num_blocks) are skipped and set
 * PKV_DEVERR_PAIR.  Destinations must be distinct.
 */
pkv_status pkv_swap_blocks(const void* src_k_pool, const void* src_v_pool, int src_num_blocks,
                           void* dst_k_pool, void* dst_v_pool, int dst_num_blocks, size_t block_bytes,
                           const int64_t* pairs, int num_pairs, uint32_t* device_error, void* stream);

/*
 * Host-side check of the preconditions of pkv_copy_blocks and pkv_swap_blocks
 * (glossary "PagedAttention", section "Sharing blocks across sequences": a
 * copy-on-write gives the writer a block of its own), which the kernels cannot
 * check without a synchronisation: pairs is int64 [num_pairs][2] (src, dst) in
 * HOST memory; every src in [0, src_num_blocks), every dst in
 * [0, dst_num_blocks), the destinations distinct and, when same_pool is
 * non-zero (a copy within one pool), no destination also a source.  Returns
 * PKV_OK or PKV_ERR_INVALID_ARG; reads pairs only, launches nothing, keeps no
 * state.  The Python binding runs it before those calls when asked to (or
 * when the environment variable PKV_DEBUG is set).
 */
pkv_status pkv_check_block_pairs(const int64_t* pairs, int num_pairs, int src_num_blocks,
                                 int dst_num_blocks, int same_pool);

/*
 * Host-side block manager (no GPU involved): the bookkeeping that produces block
 * tables, slot mappings and copy-on-write pairs for the kernels above
 * (glossary "PagedAttention", sections "How paging works" and "Sharing blocks
 * across sequences").  Blocks are handed out from a FIFO free list; a sequence
 * takes a new block only when its last one is full; a fork shares every block of
 * its parent (reference counts); appending to a partially filled block that other
 * sequences still reference first moves the writer to a fresh block and reports
 * the (src, dst) copy for pkv_copy_blocks -- the last holder writes in place;
 * freeing a sequence returns blocks whose count drops to zero to the back of the
 * free list.  All arrays are HOST memory.  Calls on one manager are serialised
 * internally (thread-safe).  A call that fails returns a status and changes
 * nothing.
 */
typedef struct pkv_block_manager pkv_block_manager;

/* free_order: a permutation of 0..num_blocks-1 giving the initial free-list order
 * (NULL = ascending).  Returns NULL for invalid arguments or memory exhaustion. */
pkv_block_manager* pkv_bm_create(int num_blocks, int block_size, const int32_t* free_order);
void pkv_bm_destroy(pkv_block_manager* m);
int pkv_bm_num_free(pkv_block_manager* m);
/* A new empty sequence; PKV_ERR_INVALID_ARG if seq_id exists. */
pkv_status pkv_bm_add_sequence(pkv_block_manager* m, int64_t seq_id);
/* child starts as a copy of parent's table and length, sharing every block. */
pkv_status pkv_bm_fork(pkv_block_manager* m, int64_t parent, int64_t child);
/* Append one token to each of the n distinct sequences, in order: slots[i] is the
 * slot (block_id * block_size + offset) where sequence i's new token goes; copy
 * pairs (int64 [max_pairs][2], src then dst) are written for shared partial
 * blocks and their count stored in *num_pairs.  PKV_ERR_OUT_OF_BLOCKS if the free
 * list is too short (nothing changes: the caller may free or preempt and retry). */
pkv_status pkv_bm_append_slots(pkv_block_manager* m, const int64_t* seq_ids, int n, int64_t* slots,
                               int64_t* pairs, int max_pairs, int* num_pairs);
/* Append n tokens to one sequence (a prefill chunk): slots[0..n) receive the
 * tokens' slots in order; a shared partially filled last block is copied once
 * before the first write (one (src, dst) pair, *num_pairs = 1, else 0), and the
 * tokens beyond it take new blocks.  The same result as n calls of
 * pkv_bm_append_slots for this sequence alone.  PKV_ERR_OUT_OF_BLOCKS if the
 * free list is too short (nothing changes). */
pkv_status pkv_bm_append_tokens(pkv_block_manager* m, int64_t seq_id, int n, int64_t* slots,
                                int64_t* pairs, int max_pairs, int* num_pairs);
/* Drop a sequence; its blocks' reference counts fall, unreferenced blocks return. */
pkv_status pkv_bm_free_sequence(pkv_block_manager* m, int64_t seq_id);
/* Rows of int32 [n][max_blocks] block tables (entries past a sequence's last block
 * set to pad) and, if context_lens is not NULL, the sequences' lengths. */
pkv_status pkv_bm_block_tables(pkv_block_manager* m, const int64_t* seq_ids, int n, int32_t* tables,
                               int max_blocks, int32_t pad, int32_t* context_lens);
int pkv_bm_ref_count(pkv_block_manager* m, int32_t block);          /* -1 if out of range */
int64_t pkv_bm_sequence_length(pkv_block_manager* m, int64_t seq_id);  /* -1 if unknown */

/* Prefix caching by block content (glossary, section "Sharing blocks across
 * sequences": hashing whole blocks extends sharing across requests; "Paged
 * Attention" study notes, section on prefix caching: look up by hash, then
 * confirm the prefix matches).  pkv_bm_cache_sequence registers the full blocks
 * covering tokens[0 .. num_tokens) of an existing sequence (num_tokens <= its
 * length) under a hash chained over each block's token ids and its
 * predecessor's hash.  pkv_bm_add_sequence_cached creates a sequence for a
 * prompt of num_tokens token ids: its leading full blocks that hit the cache --
 * same tokens, same predecessor, confirmed exactly, at most (num_tokens - 1) /
 * block_size blocks so that at least one token is left to compute -- are shared
 * (reference counts), and *num_cached_tokens receives their token count (the
 * sequence's length); the caller appends and prefills the rest.  Registered
 * blocks that no sequence holds stay cached until the free list runs dry, then
 * the one released longest ago is reused (pkv_bm_num_free counts them as free).
 * pkv_bm_num_cached: registered blocks. */
pkv_status pkv_bm_add_sequence_cached(pkv_block_manager* m, int64_t seq_id, const int32_t* tokens, int num_tokens,
                                      int* num_cached_tokens);
pkv_status pkv_bm_cache_sequence(pkv_block_manager* m, int64_t seq_id, const int32_t* tokens, int num_tokens);
int pkv_bm_num_cached(pkv_block_manager* m);

/* Move sequences between two managers with the same block size (e.g. a GPU
 * pool's and a host pool's, for preemption by swapping): every distinct block
 * the n sequences use in `from` gets one block in `to`; the sequences leave
 * `from` (their references drop there) and appear in `to` with the same
 * lengths and correspondingly shared blocks.  The (from block, to block) pairs,
 * int64 [max_pairs][2], feed pkv_swap_blocks; *num_pairs receives their count.
 * PKV_ERR_OUT_OF_BLOCKS if `to` is short of blocks (nothing changes). */
pkv_status pkv_bm_swap(pkv_block_manager* from, pkv_block_manager* to, const int64_t* seq_ids, int n,
                       int64_t* pairs, int max_pairs, int* num_pairs);

/*
 * Diagnostic for the failure handling above (no counterpart on the pages): runs one
 * kernel whose single wait can never be satisfied; the wait gives up after
 * timeout_us microseconds (1 .. 10,000,000) and OR-s PKV_DEVERR_TIMEOUT into
 * *device_error (device pointer, required).  Nothing faults or hangs; the
 * context stays usable.  A decode call given a device_error word that already
 * holds PKV_DEVERR_TIMEOUT finishes at once and writes NaN (a grid that saw a
 * wait give up stops early), so clear the word after reading it.
 */
pkv_status pkv_selftest_bounded_wait(uint32_t* device_error, unsigned timeout_us, void* stream);

/*
 * Measurement helper (no counterpart on the pages): reads every byte of a device
 * buffer once and discards it, the read-only HBM rate that a read-mostly kernel
 * such as pkv_paged_attn_decode can be held against (a copy's rate counts
 * writes too).  buf: device pointer, 16-byte aligned; bytes: a multiple of 16;
 * sink: device uint32 word, may be NULL (it is only written in the practically
 * impossible case that the folded data equal a fixed constant, which keeps the
 * loads from being optimised away).  Asynchronous on stream; PKV_ERR_ALIGNMENT
 * for a misaligned buffer or size.
 */
pkv_status pkv_stream_read(const void* buf, size_t bytes, uint32_t* sink, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* PAGEDKV_H */
