/*
 * libpagedattn: paged KV cache decode attention for NVIDIA B200 (sm_100a).
 *
 * The KV cache is split into fixed-size physical blocks; each sequence reaches
 * its blocks through a block table. This library provides the three device
 * operations of a decode step and the host-side block manager that feeds them.
 *
 * Page tags used in citations:
 *   P1 = "Paged Attention：大模型推理显存优化的核心方案" (learnblockchain.cn)
 *   P2 = "PagedAttention：操作系统级 KV 缓存虚拟内存管理" (freeguideonline.com)
 *   P3 = "PagedAttention 和 vLLM" (aiunderstanding.org)
 *
 * Conventions for every entry point:
 *   - Every call returns a pa_status; nothing is thrown across the ABI.
 *   - Device operations are asynchronous on `stream` (a cudaStream_t passed as
 *     void*; NULL is the legacy default stream). Arguments are checked on the
 *     host before launch (PA_ERR_INVALID_ARG / PA_ERR_UNSUPPORTED, nothing is
 *     launched). A failed launch returns PA_ERR_CUDA. Problems that only the
 *     device can see (a block id or slot outside the pool, a context length
 *     above its stated bound) make the kernel skip the access and record the
 *     first such event in a per-device error word that pa_get_device_error
 *     reads; the kernels never trap.
 *   - All device pointers are owned by the caller, must be 16-byte aligned and
 *     must stay valid until the stream has executed the call. The library
 *     allocates no device memory.
 *   - KV cache layout: K and V are each [num_blocks][num_kv_heads][block_size]
 *     [head_dim], row-major, in the cache dtype. Token t of a sequence is at
 *     block block_table[t / block_size], offset t % block_size (P2 §2.3, §五).
 *     A "slot" is block * block_size + offset.
 *   - Query head h reads kv head h / (num_q_heads / num_kv_heads).
 *   - Supported shapes: head_dim 64 or 128; block_size 1, 2, 4, 8, 16 or 32;
 *     num_q_heads / num_kv_heads in {1, 2, 4, 8}; dtype fp32, bf16, or 8-bit
 *     e4m3 / int8 (every operation; fp32 has no prefill and no shared-prefix
 *     decode).
 */
#ifndef PAGEDATTN_H
#define PAGEDATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  PA_OK = 0,
  PA_ERR_INVALID_ARG = 1,     /* null / misaligned pointer, negative size, bad layout */
  PA_ERR_UNSUPPORTED = 2,     /* shape or dtype outside the supported set */
  PA_ERR_NO_FREE_BLOCKS = 3,  /* block manager: the pool cannot satisfy the call */
  PA_ERR_UNKNOWN_SEQ = 4,     /* block manager: no such sequence id */
  PA_ERR_SEQ_EXISTS = 5,      /* block manager: the sequence id is already live */
  PA_ERR_CUDA = 6,            /* a CUDA runtime call or a launch failed */
  PA_ERR_DEVICE_BOUNDS = 7,   /* a kernel met an index outside its bounds and skipped it */
  PA_ERR_DEVICE_TIMEOUT = 8   /* a kernel gave up a bounded wait on its own copies */
} pa_status;

/* Cache element types. PA_FP8_E4M3 stores K and V as 8-bit floats (e4m3,
 * no infinities, largest 448), PA_INT8 as integers in [-127, 127], each with
 * one scale per tensor (pa_cache.k_scale, v_scale): element = code * scale.
 * The q/k/v inputs of an 8-bit cache are bf16;
 * the decode and the prefill round q to f16 for their tensor-core products, so
 * |q| must stay below 65504 (bf16 values from 2^-17 up to that convert exactly;
 * smaller ones move by at most 2^-25). */
typedef enum { PA_F32 = 0, PA_BF16 = 1, PA_FP8_E4M3 = 2, PA_INT8 = 3 } pa_dtype;

typedef void* pa_stream; /* cudaStream_t */

typedef struct pa_bm pa_bm; /* host block manager handle (see below) */

/* A paged KV cache in device memory (see the layout above). */
typedef struct {
  void* k;               /* device, [num_blocks][num_kv_heads][block_size][head_dim] */
  void* v;               /* device, same shape as k */
  int64_t num_blocks;    /* physical blocks in the pool, >= 1, < 2^31 */
  int32_t num_kv_heads;  /* >= 1 */
  int32_t block_size;    /* tokens per block */
  int32_t head_dim;      /* elements per head row */
  int32_t dtype;         /* pa_dtype of k, v (and of the q/k/v inputs, bf16 for 8-bit) */
  float k_scale;         /* 8-bit dtypes only: K element = code * k_scale (> 0) */
  float v_scale;         /* 8-bit dtypes only: V element = code * v_scale (> 0) */
} pa_cache;

/* Human-readable name of a status code (static storage). */
const char* pa_status_string(pa_status status);

/* Library ABI version, currently 1. */
int32_t pa_version(void);

/* ------------------------------------------------------------------------- */
/* Device operations                                                          */
/* ------------------------------------------------------------------------- */

/*
 * KV append: write each new token's K and V rows into its slot.
 * P2 §3.2.2 step 3 (write the new K, V at the block position) and §3.2.1
 * (a prompt's K, V written into its blocks).
 *
 *   k, v          device, [num_tokens][num_kv_heads][head_dim], cache dtype,
 *                 contiguous.
 *   slot_mapping  device int64 [num_tokens]; slot of token i, or -1 to skip it.
 *                 A slot outside [-1, num_blocks * block_size) is skipped and
 *                 recorded as PA_ERR_DEVICE_BOUNDS.
 *   num_tokens    >= 0; 0 launches nothing.
 * Two tokens must not name the same slot in one call (the result would be
 * either row). A bit copy for fp32 / bf16 caches. For an 8-bit cache the
 * rows are bf16 and each element is stored as the code of x / scale computed
 * in fp32 and rounded to nearest even: e4m3 clamped to +-448 (NaN stays NaN),
 * int8 clamped to [-127, 127] (NaN becomes 0) (the "quantised code" step of
 * an 8-bit KV cache).
 */
pa_status pa_reshape_and_cache(const void* k, const void* v, const int64_t* slot_mapping, int32_t num_tokens,
                               const pa_cache* cache, pa_stream stream);

/*
 * Copy whole physical blocks, K and V: cache[dst] = cache[src] for each pair.
 * P2 §3.4: before a write into a block shared by several sequences, the block
 * is copied and the writer's table is pointed at the copy (copy-on-write).
 *
 *   src_dst_pairs  device int32 [n_pairs][2] = {src, dst}.
 *   n_pairs        >= 0; 0 launches nothing.
 * All dst must differ, and no dst may be the src of another pair in the same
 * call (the pairs that pa_bm_append_slot(s) emits satisfy this). An id outside
 * [0, num_blocks) skips that pair and is recorded as PA_ERR_DEVICE_BOUNDS.
 * Apply the pairs of a decode step before the pa_reshape_and_cache that writes
 * the step's tokens, on the same stream.
 */
pa_status pa_copy_blocks(const pa_cache* cache, const int32_t* src_dst_pairs, int32_t n_pairs, pa_stream stream);

/*
 * Swap whole blocks between the device pool and a host pool (P2 §五 page
 * replacement: inactive blocks move to CPU memory when the GPU runs short;
 * P2 §八 GPU/CPU tiers).
 *
 *   host_k, host_v   host pools [host_num_blocks][num_kv_heads][block_size]
 *                    [head_dim] in the cache dtype, in pinned memory mapped
 *                    into the device's address space (cudaHostAlloc, or
 *                    cudaHostRegister with mapping); anything else returns
 *                    PA_ERR_INVALID_ARG before launch.
 *   pairs            device int32 [n_pairs][2]: {device block, host block} when
 *                    to_host != 0 (swap out), {host block, device block}
 *                    otherwise (swap in), as pa_bm_swap_out / pa_bm_swap_in
 *                    emit them. Ids out of range skip the pair and are recorded
 *                    as PA_ERR_DEVICE_BOUNDS.
 * One kernel moves every pair (no per-block copy calls). Run it before any
 * later write reuses the released blocks, on the same stream.
 */
pa_status pa_swap_blocks(const pa_cache* cache, void* host_k, void* host_v, int64_t host_num_blocks,
                         const int32_t* pairs, int32_t n_pairs, int32_t to_host, pa_stream stream);

/*
 * pa_swap_blocks on the copy engines: the same move, with the pairs in host
 * memory and one cudaMemcpyAsync per tensor for every run of pairs whose
 * source and destination ids both advance by one (a single block when the ids
 * are scattered). host_k, host_v: pinned host pools (cudaHostAlloc or
 * cudaHostRegister; no device mapping needed). Ids are checked on the host
 * before any copy (PA_ERR_INVALID_ARG). Leaves the SMs free; costs one host
 * call per run.
 */
pa_status pa_swap_blocks_copy(const pa_cache* cache, void* host_k, void* host_v, int64_t host_num_blocks,
                              const int32_t* host_pairs, int32_t n_pairs, int32_t to_host, pa_stream stream);

/*
 * Single-query decode attention over the paged cache.
 * P2 §1.1: out = softmax(scale * q K^T) V, one query row per head; P2 §3.2.2
 * step 4 and §4.1: every logical block of the sequence is visited through its
 * block table, with the softmax accumulated block by block (online softmax).
 *
 *   q                  device, [num_seqs][num_q_heads][head_dim], cache dtype.
 *   block_tables       device int32 [num_seqs][max_blocks_per_seq]; entries
 *                      past ceil(context_len / block_size) are never read.
 *   context_lens       device int32 [num_seqs]; tokens to attend over,
 *                      including the token appended this step. Must not
 *                      exceed max_context_len (larger values are clamped and
 *                      recorded as PA_ERR_DEVICE_BOUNDS). 0 gives a zero row.
 *   max_context_len    host bound on context_lens, <= max_blocks_per_seq *
 *                      block_size; it sizes the launch.
 *   scale              score scale, usually 1/sqrt(head_dim).
 *   out                device fp32 [num_seqs][num_q_heads][head_dim].
 *   partition_tokens   0: one CTA walks the whole sequence.
 *                      > 0 (a multiple of block_size): split each sequence
 *                      into partitions of that many tokens, each computed
 *                      separately; a second kernel merges them with a
 *                      log-sum-exp reduction.
 *                      -1: chosen by the library (pa_decode_partition_tokens).
 *   workspace          device, >= pa_decode_workspace_bytes(...) bytes,
 *                      256-byte aligned. Always needed: it holds the work
 *                      counters of the persistent kernels (cleared by the call
 *                      itself) and, when sequences are split, the partial
 *                      results. Its contents need no initial value.
 * Accumulation is fp32. Calls sharing a workspace must not overlap on the GPU.
 */
pa_status pa_decode(const void* q, int32_t num_seqs, int32_t num_q_heads, const pa_cache* cache,
                    const int32_t* block_tables, int32_t max_blocks_per_seq, const int32_t* context_lens,
                    int32_t max_context_len, float scale, float* out, int32_t partition_tokens, void* workspace,
                    size_t workspace_bytes, pa_stream stream);

/*
 * pa_decode with a dispatch order: sequence seq_order[y] is served by grid
 * row y (and, in the persistent kernels, by the items of row y), so passing
 * the rows longest first (pa_bm_longest_first) starts the long CTAs in the
 * first waves and leaves the short ones for the end. Results are those of
 * pa_decode, bit for bit.
 *   seq_order  device int32 [num_seqs], a permutation of 0 .. num_seqs-1,
 *              4-byte aligned (NULL: batch order). An entry out of range is
 *              recorded as PA_ERR_DEVICE_BOUNDS (pa_get_device_error) and its
 *              row served in batch order; a repeated entry leaves some
 *              sequence uncomputed (no memory outside the arguments is
 *              touched).
 * Other arguments, supported shapes and errors as pa_decode.
 */
pa_status pa_decode_ordered(const void* q, int32_t num_seqs, int32_t num_q_heads, const pa_cache* cache,
                            const int32_t* block_tables, int32_t max_blocks_per_seq, const int32_t* context_lens,
                            int32_t max_context_len, const int32_t* seq_order, float scale, float* out,
                            int32_t partition_tokens, void* workspace, size_t workspace_bytes, pa_stream stream);

/*
 * One decode step in one launch: the KV append (pa_reshape_and_cache of each
 * sequence's new token, P2 §3.2.2 step 3) fused into pa_decode_ordered (step
 * 4). The CTA (or persistent work item) that covers sequence s's last token
 * first writes, for its kv head, the new K and V rows at slot_mapping[s] and
 * only then starts the copies that read that block; no other CTA of the launch
 * reads that position. Results and cache contents are those of
 * pa_reshape_and_cache followed by pa_decode, bit for bit.
 *   k_new, v_new   device [num_seqs][num_kv_heads][head_dim], 16-byte aligned:
 *                  bf16 for a bf16 or 8-bit cache (quantised with the cache's
 *                  k_scale / v_scale as pa_reshape_and_cache does), fp32 for
 *                  an fp32 cache.
 *   slot_mapping   device int64 [num_seqs], 8-byte aligned: the slot of each
 *                  sequence's new token, which must be its position
 *                  context_lens[s] - 1 in its block table (as
 *                  pa_bm_append_slots returns it); -1 writes nothing. The
 *                  target block must not be shared (run pa_copy_blocks for the
 *                  step's copy-on-write pairs first, on the same stream). A
 *                  slot outside the pool is recorded as PA_ERR_DEVICE_BOUNDS
 *                  and not written.
 * Other arguments, supported shapes and errors as pa_decode_ordered
 * (seq_order may be NULL). Not for the cascade (pa_decode_cascade): append
 * first there.
 */
pa_status pa_decode_append(const void* q, const void* k_new, const void* v_new, const int64_t* slot_mapping,
                           int32_t num_seqs, int32_t num_q_heads, const pa_cache* cache, const int32_t* block_tables,
                           int32_t max_blocks_per_seq, const int32_t* context_lens, int32_t max_context_len,
                           const int32_t* seq_order, float scale, float* out, int32_t partition_tokens,
                           void* workspace, size_t workspace_bytes, pa_stream stream);

/*
 * Causal attention of newly written prompt tokens (prefill, possibly in
 * chunks) over the paged cache. P2 §3.2.1: the prompt's K, V are computed and
 * written into the sequence's blocks (pa_reshape_and_cache first); each new
 * token attends, through the block table, to every position of its sequence up
 * to and including its own (P2 §1.1 formula, §2.3 table walk).
 *
 *   q              device bf16 [T][num_q_heads][head_dim], the new tokens of
 *                  all sequences back to back (T = cu_q_lens[num_seqs]).
 *   cu_q_lens      device int32 [num_seqs + 1]: sequence s owns rows
 *                  cu_q_lens[s] .. cu_q_lens[s+1]-1; n_s = their count.
 *   max_q_len      host bound on every n_s; it sizes the launch, and
 *                  num_seqs * max_q_len bounds the rows the kernel's
 *                  tensor-memory copies of q and out may address (only rows of
 *                  query tiles lying wholly inside their sequence are copied
 *                  that way, so every row they touch exists).
 *   context_lens   device int32 [num_seqs]: length L_s including the new
 *                  tokens; new token i of s sits at position L_s - n_s + i and
 *                  sees positions 0 .. L_s - n_s + i. n_s > L_s or L_s above
 *                  max_context_len is clamped and recorded (PA_ERR_DEVICE_BOUNDS).
 *   out            device fp32 [T][num_q_heads][head_dim].
 * q and out must be 16-byte aligned (PA_ERR_INVALID_ARG otherwise).
 * Supported: bf16, e4m3 or int8 cache, block_size >= 8 (16, 32 as for decode),
 * head_dim 64 or 128, num_q_heads / num_kv_heads in {1, 2, 4, 8}; fp32 caches
 * return PA_ERR_UNSUPPORTED. Accumulation is fp32 on the tensor cores. The
 * softmax weights enter the P V product as f16 (11 significant bits, weights
 * at most 2^8), so V is read as f16: over a bf16 cache each V element is
 * converted on chip, exactly for |v| in [2^-14, 65504] (smaller values move by
 * less than 2^-25; |v| above 65504 is out of range); q and K stay bf16 for the
 * q K^T product. Over an 8-bit cache the codes are widened to f16 (exactly)
 * and q is rounded to f16.
 */
pa_status pa_prefill(const void* q, int32_t num_seqs, const int32_t* cu_q_lens, int32_t max_q_len, int32_t num_q_heads,
                     const pa_cache* cache, const int32_t* block_tables, int32_t max_blocks_per_seq,
                     const int32_t* context_lens, int32_t max_context_len, float scale, float* out, pa_stream stream);

/*
 * Decode with shared prefixes read once per group (P2 §3.4: sequences sharing
 * a prefix point at the same physical blocks; P1 "跨请求的内存共享": parallel
 * samples of one prompt). Same result as pa_decode, computed in three parts:
 * for each group, one pass over the shared prefix blocks attends all members'
 * queries at once (rows = members x query heads on the tensor cores); each
 * sequence's own suffix [seq_prefix_tokens[s], L_s) goes through the decode
 * kernels; a log-sum-exp merge combines them (done by the suffix CTA itself
 * when sequences are not split into partitions, else by a merge kernel).
 * Prefix K/V bytes are read once per group instead of once per member.
 *
 *   group_offsets        device int32 [num_groups + 1]; group j's members are
 *                        group_members[group_offsets[j] .. group_offsets[j+1]).
 *   group_members        device int32: sequence indices (0 .. num_seqs-1), each
 *                        in at most one group; at most 64 / (num_q_heads /
 *                        num_kv_heads) members per group (max_group_size).
 *   group_prefix_tokens  device int32 [num_groups]: tokens shared by every
 *                        member (identical physical blocks, read through the
 *                        first member's table), a multiple of 64.
 *   seq_prefix_tokens    device int32 [num_seqs]: its group's prefix length,
 *                        0 for a sequence in no group.
 *   max_prefix_tokens    host bound on group_prefix_tokens.
 *   seq_order            device int32 [num_seqs] or NULL: the order in which
 *                        the sequences' suffix CTAs are dispatched, a
 *                        permutation of 0 .. num_seqs-1 (pa_bm_longest_first
 *                        puts the longest suffixes first, so that the long
 *                        CTAs start in the first waves and the short ones
 *                        fill the end). Results do not depend on it. An entry
 *                        out of range is recorded as PA_ERR_DEVICE_BOUNDS (see
 *                        pa_get_device_error) and its row is served in batch
 *                        order; a repeated entry leaves some sequence
 *                        uncomputed (no memory outside the arguments is
 *                        touched).
 *   workspace            >= pa_decode_cascade_workspace_bytes(...).
 * Other arguments as pa_decode (partition size chosen by the library).
 * Supported: bf16, e4m3 or int8 cache, block_size 8..32; other shapes return
 * PA_ERR_UNSUPPORTED. Over an 8-bit cache the prefix pass widens the codes to
 * f16 in shared memory and multiplies by f16 weights (as pa_prefill does).
 */
pa_status pa_decode_cascade(const void* q, int32_t num_seqs, int32_t num_q_heads, const pa_cache* cache,
                            const int32_t* block_tables, int32_t max_blocks_per_seq, const int32_t* context_lens,
                            int32_t max_context_len, int32_t num_groups, const int32_t* group_offsets,
                            const int32_t* group_members, const int32_t* group_prefix_tokens,
                            const int32_t* seq_prefix_tokens, int32_t max_group_size, int32_t max_prefix_tokens,
                            const int32_t* seq_order, float scale, float* out, void* workspace,
                            size_t workspace_bytes, pa_stream stream);

size_t pa_decode_cascade_workspace_bytes(int32_t num_seqs, int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                                         int32_t max_context_len, int32_t block_size, int32_t max_prefix_tokens);

/* The partition size pa_decode uses for partition_tokens = -1 with these
 * sizes (0 = no split). */
int32_t pa_decode_partition_tokens(int32_t num_seqs, int32_t num_q_heads, int32_t num_kv_heads,
                                   int32_t max_context_len, int32_t block_size);

/* The same for pa_decode_ordered / pa_decode_append with a seq_order (the
 * CTAs dispatched longest first balance the waves, so fewer splits pay):
 * never more partitions than pa_decode_partition_tokens gives, so
 * pa_decode_workspace_bytes(..., -1) covers it. */
int32_t pa_decode_ordered_partition_tokens(int32_t num_seqs, int32_t num_q_heads, int32_t num_kv_heads,
                                           int32_t max_context_len, int32_t block_size);

/* Workspace bytes pa_decode needs for these sizes (a few hundred bytes of
 * counters, plus the partials when sequences are split). partition_tokens may
 * be -1 (resolved as pa_decode would). */
size_t pa_decode_workspace_bytes(int32_t num_seqs, int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                                 int32_t max_context_len, int32_t block_size, int32_t partition_tokens);

/*
 * Waits for `stream`, then reads and clears this device's error word.
 * Returns PA_OK, PA_ERR_DEVICE_BOUNDS or PA_ERR_DEVICE_TIMEOUT (the first event
 * recorded since the last read), or PA_ERR_CUDA. `info_out` (may be NULL)
 * receives the offending value (block id, slot or length) when there is one.
 */
pa_status pa_get_device_error(pa_stream stream, int64_t* info_out);

/* Bytes of the fixed device array behind pa_decode_static_workspace. */
#define PA_STATIC_WORKSPACE_BYTES (16u << 20)

/*
 * pa_decode without a caller-provided workspace, for callers that cannot
 * allocate device memory. The pages have no counterpart: this is a deployment
 * variant of pa_decode. Some hosts hand an attention kernel only its inputs
 * and outputs: an inference runtime that reserves the whole device up front
 * and gives plug-ins no workspace, or a latency-bound serving loop where a
 * cudaMalloc (which may synchronise the device) is not allowed between steps.
 * Arguments, results and errors are those of pa_decode; the workspace pa_decode
 * would take (its work counters and the partial results of split sequences)
 * is an array of PA_STATIC_WORKSPACE_BYTES compiled into the library, which
 * every device that loads the library holds until the process exits. Every
 * call with num_seqs > 0 uses the array (the counters at least, whatever
 * partition_tokens is). A call whose need (pa_decode_workspace_bytes) is
 * larger than the array returns PA_ERR_INVALID_ARG and launches nothing.
 * The first such call on each device looks up that device's address of the
 * array and keeps it; make that first call before any stream capture. The
 * kept address is not refreshed, so the library must not outlive a reset of
 * the device (cudaDeviceReset) in the same process. The array is shared by
 * every call on the device and keeps the last call's contents; nothing in it
 * needs an initial value. Calls that overlap on the GPU (other streams, other
 * threads) race on the array and must be serialised by the caller.
 * Allocates nothing: no cudaMalloc, cudaFree or allocating library call.
 */
pa_status pa_decode_static_workspace(const void* q, int32_t num_seqs, int32_t num_q_heads, const pa_cache* cache,
                                     const int32_t* block_tables, int32_t max_blocks_per_seq,
                                     const int32_t* context_lens, int32_t max_context_len, float scale, float* out,
                                     int32_t partition_tokens, pa_stream stream);

/*
 * One whole decode step from host memory: the call a serving loop makes per
 * generated token. P2 §3.2.2 steps 1-4 in order: for each listed sequence the
 * block manager assigns the new token's slot (new block or copy-on-write as
 * in pa_bm_append_slots); the CoW pairs, slots, block tables and lengths are
 * staged in pinned host memory and sent in one copy; q, k, v are copied from
 * the caller's host buffers; pa_copy_blocks and pa_decode_append (the KV
 * append done by the decode CTAs) run on `stream`; the fp32 output is copied
 * back to out_host; the call returns after the stream has finished (so
 * out_host is ready).
 *
 *   bm, cache       the sequences' manager and cache (same block_size).
 *   seq_ids         host int64 [n]: sequences appending one token each.
 *   q_host          host [n][num_q_heads][head_dim], cache dtype.
 *   k_host, v_host  host [n][num_kv_heads][head_dim], cache dtype.
 *   out_host        host fp32 [n][num_q_heads][head_dim].
 *   partition_tokens as for pa_decode.
 *   dev_staging     device, >= *dev_bytes of pa_step_staging_bytes, 256-byte aligned.
 *   host_staging    pinned host, >= *host_bytes of pa_step_staging_bytes.
 * Host buffers should be pinned for asynchronous copies (pageable memory works
 * but is copied synchronously by the driver). seq_ids must be distinct. The
 * staging sizes are checked against the lengths the step produces before
 * anything changes: too-small staging (PA_ERR_INVALID_ARG) or a block-manager
 * failure (PA_ERR_NO_FREE_BLOCKS, PA_ERR_UNKNOWN_SEQ) leaves the manager
 * unchanged and launches nothing. The staging buffers are reused by the next
 * call; the call returns only after the stream has drained.
 * A batch of 16 or more sequences is cut into two row chunks whose copies,
 * appends and decodes run as separate chains on streams the library creates
 * once per device (kept until the process exits): the copy engines move one
 * chunk's inputs or outputs while the other computes. The
 * chains start after the work already queued on `stream`, and `stream` waits
 * for all of them, so the call's ordering against the caller's stream is that
 * of a single chain. Each chain's pa_decode_append dispatches its rows
 * longest first (the order changes no result bit).
 */
pa_status pa_step_host(pa_bm* bm, const pa_cache* cache, int32_t n, const int64_t* seq_ids, int32_t num_q_heads,
                       const void* q_host, const void* k_host, const void* v_host, float scale, float* out_host,
                       int32_t partition_tokens, void* dev_staging, size_t dev_staging_bytes, void* host_staging,
                       size_t host_staging_bytes, pa_stream stream);

/* Host wall-clock phases of the calling thread's last successful
 * pa_step_host call, in microseconds (all zero after a failed call): the
 * block-manager work (argument checks, slots, copy-on-write pairs, tables),
 * enqueueing the metadata copy and the copy-on-write block copies,
 * enqueueing the row chunks' chains (q/k/v copies, append, decode, output
 * copy), and the wait for the stream; total_us spans the whole call; chunks is
 * the number of row chunks the batch was cut into. The device runs the copies
 * and kernels between the first enqueue and the end of the wait. */
typedef struct {
  double block_manager_us;
  double metadata_enqueue_us;
  double chains_enqueue_us;
  double wait_us;
  double total_us;
  int32_t chunks;
} pa_step_timing;

pa_status pa_step_host_last_timing(pa_step_timing* out);

/* Staging sizes pa_step_host needs for up to n sequences whose lengths stay
 * at most max_context_len after the step. */
pa_status pa_step_staging_bytes(int32_t n, int32_t num_q_heads, const pa_cache* cache, int32_t max_context_len,
                                int32_t partition_tokens, size_t* dev_bytes, size_t* host_bytes);

/*
 * Self-test of the device wait limit. Every pipelined kernel waits for its own
 * copies with a bounded wait; this launches one thread that waits on a barrier
 * nothing completes. After timeout_ns (1 .. 10^10) it records
 * PA_ERR_DEVICE_TIMEOUT in the error word and exits, leaving the context
 * usable. Read the result with pa_get_device_error.
 */
pa_status pa_selftest_wait_timeout(int64_t timeout_ns, pa_stream stream);

/* ------------------------------------------------------------------------- */
/* Host block manager                                                         */
/* ------------------------------------------------------------------------- */
/*
 * The pool's free list, reference counts and per-sequence block tables
 * (P1 "Paged Attention 的工作原理", "块表（Block Table）"; P2 §2.3, §3.2, §3.3,
 * §3.4). Not thread-safe: one thread per handle. Every call either succeeds or
 * leaves the state unchanged.
 * Free-list order: allocation takes the front; a block whose count drops to
 * zero is appended at the back, in the order of the freed sequence's table.
 * Sequences are identified by caller-chosen int64 ids.
 */
/* free_order: host int32 [num_blocks], a permutation of 0..num_blocks-1 giving
 * the initial free-list order, or NULL for 0, 1, 2, ... */
pa_status pa_bm_create(int64_t num_blocks, int32_t block_size, const int32_t* free_order, pa_bm** out);
void pa_bm_destroy(pa_bm* bm);

/* Prefill (P2 §3.2.1): new sequence of num_tokens >= 0 tokens, given
 * ceil(num_tokens / block_size) blocks. slots_out (host int64 [num_tokens],
 * may be NULL) receives the slot of each token. */
pa_status pa_bm_add_seq(pa_bm* bm, int64_t seq_id, int32_t num_tokens, int64_t* slots_out);

/* Prefill with prefix reuse (P2 §3.4 prefix block pool; P3: cached system
 * prompts shared across requests). tokens: host int32 [num_tokens], the
 * prompt's token ids. Whole prompt blocks are matched, from block 0 on, against
 * a prefix cache keyed by the full token prefix up to each block's end; hits
 * map onto the cached blocks (one more reference each) and the rest are new
 * blocks, whose whole ones are added to the cache. slots_out (host int64
 * [num_tokens], may be NULL) gets -1 for the *n_cached_out leading tokens
 * already in the pool (pa_reshape_and_cache skips them) and the slot of every
 * other token. The cache holds one reference per listed block; a listed block
 * that only the cache holds is evictable, and any allocation of this manager
 * takes the least recently released evictable block when the free list is
 * empty. Keys are 64-bit hash chains whose block tokens and parent are checked
 * on a hit, so a false hit needs a 64-bit collision of two different prefixes. */
pa_status pa_bm_add_seq_cached(pa_bm* bm, int64_t seq_id, const int32_t* tokens, int32_t num_tokens,
                               int64_t* slots_out, int32_t* n_cached_out);

/* Host blocks available for swapping (P2 §五): ids 0..num_host_blocks-1 on a
 * FIFO free list. Fails (PA_ERR_INVALID_ARG) while a sequence is swapped out. */
pa_status pa_bm_set_host_blocks(pa_bm* bm, int64_t num_host_blocks);

/* Swap a live sequence out: each block of its table gets a host block and
 * releases one device reference (a block shared with a live sequence stays).
 * pairs_out (host int32 [cap][2]) gets {device, host} per logical block, in
 * order; *n_pairs_out the count. Apply with pa_swap_blocks(to_host = 1)
 * before the released device blocks are written again. The sequence keeps its
 * length but cannot append or decode until swapped in. All or nothing. */
pa_status pa_bm_swap_out(pa_bm* bm, int64_t seq_id, int32_t* pairs_out, int32_t cap, int32_t* n_pairs_out);

/* Swap a sequence back in: fresh device blocks (private, from the free list
 * or by eviction of cached blocks), pairs {host, device} in table order, host
 * blocks returned to their free list. Apply with pa_swap_blocks(to_host = 0)
 * before decoding it. All or nothing. pa_bm_free_seq on a swapped-out
 * sequence releases its host blocks. */
pa_status pa_bm_swap_in(pa_bm* bm, int64_t seq_id, int32_t* pairs_out, int32_t cap, int32_t* n_pairs_out);

/* Prefix-cache counters: listed blocks, evictable ones among them, and the
 * prompt tokens served from the cache so far. */
pa_status pa_bm_prefix_stats(const pa_bm* bm, int64_t* cached_blocks, int64_t* evictable_blocks,
                             int64_t* hit_tokens);

/* Share (P1 "跨请求的内存共享"; P2 §3.4): `child` gets a copy of `parent`'s
 * table and every block in it gains one reference. */
pa_status pa_bm_fork(pa_bm* bm, int64_t parent, int64_t child);

/* One decode-step position (P2 §3.2.2 steps 2-3, §3.4). If the last block is
 * full, a new block is appended to the table. If the target block is shared
 * (count > 1) it is replaced by a fresh block and *cow_pair_out = {old, new},
 * which must be applied with pa_copy_blocks before the token is written;
 * otherwise *cow_pair_out = {-1, -1}. cow_pair_out may be NULL only when the
 * caller knows no block is shared. */
pa_status pa_bm_append_slot(pa_bm* bm, int64_t seq_id, int64_t* slot_out, int32_t* cow_pair_out);

/* pa_bm_append_slot for n sequences in the given order, all or nothing.
 * slots_out: host int64 [n]; cow_pairs_out: host int32 [n][2], of which the
 * first *n_pairs_out are filled in order. */
pa_status pa_bm_append_slots(pa_bm* bm, int32_t n, const int64_t* seq_ids, int64_t* slots_out,
                             int32_t* cow_pairs_out, int32_t* n_pairs_out);

/* Release a finished sequence (P2 §3.3). */
pa_status pa_bm_free_seq(pa_bm* bm, int64_t seq_id);

/* The table of one sequence: up to `cap` entries into out (host int32), the
 * full table length into *n_out and the token count into *len_out (either may
 * be NULL). */
pa_status pa_bm_block_table(const pa_bm* bm, int64_t seq_id, int32_t* out, int32_t cap, int32_t* n_out,
                            int64_t* len_out);

/* Decode inputs for n sequences: out (host int32 [n][cap]) gets each table,
 * padded with `pad`; lens_out (host int32 [n]) the token counts. Fails with
 * PA_ERR_INVALID_ARG if a table is longer than cap. */
pa_status pa_bm_block_tables(const pa_bm* bm, int32_t n, const int64_t* seq_ids, int32_t* out, int32_t cap,
                             int32_t pad, int32_t* lens_out);

pa_status pa_bm_refcount(const pa_bm* bm, int32_t block, int32_t* out);

/*
 * Shared-prefix groups of a decode batch, the host side of pa_decode_cascade
 * (P2 §3.4: sequences sharing a prefix point at the same physical blocks;
 * P1 "跨请求的内存共享": parallel samples of one prompt).
 *
 *   seq_ids              host int64 [n]: the batch, in the order of its rows.
 *   max_group_size       >= 1; pass 64 / (num_q_heads / num_kv_heads) for
 *                        pa_decode_cascade.
 *   align_tokens         >= 1; prefixes are cut down to a multiple of it
 *                        (64 for pa_decode_cascade).
 *   group_offsets        host int32, at least n / 2 + 1 entries: group j owns
 *                        group_members[group_offsets[j] .. group_offsets[j+1]).
 *   group_members        host int32 [n]: batch row indices.
 *   group_prefix_tokens  host int32, at least n / 2 entries.
 *   seq_prefix_tokens    host int32 [n]: the row's group prefix, 0 if none.
 *   *n_groups_out        number of groups; *max_prefix_out (may be NULL) the
 *                        largest prefix.
 * Rule: sequences with at least one whole block are keyed by the physical id
 * of their first block (keys in order of first appearance); each key's rows,
 * in batch order, are cut into groups of at most max_group_size; a group's
 * prefix is the longest run of leading table entries identical in every
 * member, counted over the whole blocks of its shortest member, cut down to a
 * multiple of align_tokens. Groups of one member or with no prefix left are
 * dropped. Reads the manager only; PA_ERR_UNKNOWN_SEQ if an id is not live.
 */
pa_status pa_bm_prefix_groups(const pa_bm* bm, int32_t n, const int64_t* seq_ids, int32_t max_group_size,
                              int32_t align_tokens, int32_t* group_offsets, int32_t* group_members,
                              int32_t* group_prefix_tokens, int32_t* seq_prefix_tokens, int32_t* n_groups_out,
                              int32_t* max_prefix_out);

/*
 * Longest-first dispatch order of a decode batch (the seq_order argument of
 * pa_decode_cascade): a decode CTA's time grows with the tokens it reads, so
 * starting the longest first leaves the short ones to fill the last wave.
 *
 *   seq_ids      host int64 [n]: the batch, in the order of its rows.
 *   skip_tokens  host int32 [n] or NULL: tokens of each row not read by the
 *                CTA being ordered (pa_decode_cascade: seq_prefix_tokens).
 *   order        host int32 [n], written: the row indices sorted by
 *                decreasing (the sequence's tokens - skip_tokens[row]), ties
 *                in batch order.
 * Reads the manager only; PA_ERR_UNKNOWN_SEQ if an id is not live,
 * PA_ERR_INVALID_ARG for n < 0 or a missing array.
 */
pa_status pa_bm_longest_first(const pa_bm* bm, int32_t n, const int64_t* seq_ids, const int32_t* skip_tokens,
                              int32_t* order);

/* free_blocks: blocks on the free list (evictable cached blocks are not
 * counted); allocated_slots: block_size times the blocks not on the free
 * list; used_slots: slots holding a token of a live sequence (a shared block
 * counts once). allocated - used is the internal waste (P1 "内存浪费的两种形式")
 * plus the slots of evictable cached blocks. */
pa_status pa_bm_stats(const pa_bm* bm, int64_t* free_blocks, int64_t* used_slots, int64_t* allocated_slots);

/* The free list in order: up to cap ids into out, the length into *n_out. */
pa_status pa_bm_free_list(const pa_bm* bm, int32_t* out, int64_t cap, int64_t* n_out);

#ifdef __cplusplus
}
#endif

#endif /* PAGEDATTN_H */
