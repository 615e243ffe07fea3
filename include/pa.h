/*
 * pa.h - C ABI of the paged KV-cache decode library (libpagedattn.so).
 *
 * The KV cache is a pool of fixed-size physical blocks, each holding the keys
 * and values of `block_size` tokens; every sequence keeps a block table that
 * lists, in logical order, which physical blocks hold it, and the attention
 * kernel follows that table instead of assuming one unbroken stretch of
 * memory per sequence ("Paged Attention: Virtual Memory for the KV Cache", section "The fix
 * borrowed from operating systems"; glossary "Paged attention", section "What
 * is Paged Attention?").
 *
 * Four device operations:
 *   pa_write_kv    - store each new token's K and V into its slot;
 *   pa_copy_blocks - copy whole blocks: the copy-on-write step when a sequence
 *                    diverges inside a shared block;
 *   pa_swap_blocks - move whole blocks between the device pools and a pool in
 *                    host memory (preemption by swapping);
 *   pa_decode      - single-query attention of every sequence over its paged
 *                    context.
 *
 * Conventions for every call:
 *   - All array pointers are caller-owned DEVICE memory (in practice PyTorch
 *     tensors). The library never allocates, frees or synchronises device
 *     memory; it only enqueues kernels on `stream` (0 = legacy default stream).
 *   - Argument checks run on the host, synchronously, before anything is
 *     enqueued; a rejected call has enqueued nothing. Errors that depend on
 *     device data are the caller's contract, but never lead to an access
 *     outside the caller's buffers: pa_write_kv / pa_copy_blocks skip slots and
 *     blocks outside the pool; pa_decode reads block 0 in place of a table
 *     entry outside the pool and writes zero rows for a sequence whose length
 *     is negative or exceeds max_context_len or its table, and records
 *     PA_ERR_INVALID_ARG in its status word (pa_decode_status).
 *   - A launch failure is reported as PA_ERR_CUDA; pa_last_cuda_error() gives
 *     the CUDA error string of the most recent such failure on this thread.
 *   - Every array must be 16-byte aligned and densely packed in the layout
 *     given (row-major, innermost index last).
 *   - Each call is wrapped in an NVTX range named after it, for timeline
 *     profilers; without one attached, that costs two function calls.
 */
#ifndef PAGED_KV_CACHE_PA_H
#define PAGED_KV_CACHE_PA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Opaque CUDA stream handle (a cudaStream_t). */
typedef void* pa_stream_t;

typedef enum {
  PA_F32 = 0,
  PA_F16 = 1,
  PA_BF16 = 2
} pa_dtype;

typedef enum {
  PA_OK = 0,
  PA_ERR_INVALID_ARG = 1,          /* null pointer, negative size, bad shape */
  PA_ERR_UNSUPPORTED = 2,          /* dtype / head_dim / block_size not built */
  PA_ERR_MISALIGNED = 3,           /* a pointer is not 16-byte aligned */
  PA_ERR_WORKSPACE_TOO_SMALL = 4,  /* see pa_decode_workspace_size */
  PA_ERR_CUDA = 5,                 /* a CUDA call failed; see pa_last_cuda_error */
  PA_ERR_DEVICE_TIMEOUT = 6        /* a kernel gave up waiting (see pa_decode_status) */
} pa_status;

/*
 * The two pools of one layer's cache, each num_blocks x num_kv_heads tiles of
 * block_size x head_dim elements of type `dtype` (the byte size of a
 * [num_blocks, num_kv_heads, block_size, head_dim] array). Slot s (a token)
 * lives in block s / block_size at offset s % block_size. Each (block, KV
 * head) tile is contiguous, tile (b, h) starting at element
 * (b * num_kv_heads + h) * block_size * head_dim. Inside a tile, rows are cut
 * into 64-element halves and grouped 16 tokens at a time: element (t, d) of
 * the tile sits at
 *   ((t / SH) * NH + d / 64) * SH * 64 + (t % SH) * 64 + d % 64,
 *   SH = min(block_size, 16), NH = head_dim / 64
 * (plain row-major when head_dim is 64). The pages leave the inside of a block
 * open; this order lets one copy of a tile feed the tensor cores. Write and
 * read the pools through pa_write_kv / pa_copy_blocks / pa_decode.
 * Supported: dtype F32/F16/BF16, head_dim 64/128, block_size 8/16/32
 * (the block sizes the pages call typical: "Paged Attention as a Memory
 * Manager", "Virtual Memory as the Blueprint").
 */
typedef struct {
  void* k_cache;
  void* v_cache;
  int32_t num_blocks;
  int32_t num_kv_heads;
  int32_t block_size;
  int32_t head_dim;
  pa_dtype dtype;
} pa_kv_cache;

/*
 * pa_write_kv - store new tokens' keys and values into their slots.
 *
 * A sequence fills its current block and takes a new one only when it needs
 * one ("The fix borrowed from operating systems"); the host decides the slot,
 * this call only stores. For token t (0 <= t < num_tokens) and KV head h:
 *   k_cache[slot / BS][h][slot % BS][:] = key[t][h][:]   (same for V)
 * with slot = slot_mapping[t]; a negative slot skips the token (padding).
 *
 *   key, value    device [num_tokens, num_kv_heads, head_dim], cache dtype
 *   slot_mapping  device int64 [num_tokens]; slots must be distinct within a
 *                 call and < num_blocks * block_size
 * Bit-exact copy. num_tokens == 0 is a no-op returning PA_OK.
 */
pa_status pa_write_kv(const pa_kv_cache* cache, const void* key,
                      const void* value, const int64_t* slot_mapping,
                      int32_t num_tokens, pa_stream_t stream);

/*
 * pa_copy_blocks - copy-on-write block copies.
 *
 * When a sequence is about to write into a block it shares, it first gets its
 * own copy of that block ("Paged Attention: Virtual Memory for the KV Cache",
 * section "Sharing comes almost for free"). For each pair p:
 *   k_cache[dst] = k_cache[src]; v_cache[dst] = v_cache[src]   (all heads)
 * with (src, dst) = (block_pairs[2p], block_pairs[2p + 1]).
 *
 *   block_pairs  device int64 [num_pairs][2]; every dst distinct and never a
 *                src in the same call (otherwise the result is order-dependent)
 * Bit-exact copy. num_pairs == 0 is a no-op returning PA_OK.
 */
pa_status pa_copy_blocks(const pa_kv_cache* cache, const int64_t* block_pairs,
                         int32_t num_pairs, pa_stream_t stream);

/* Direction of pa_swap_blocks. */
typedef enum {
  PA_SWAP_OUT = 0, /* device pools -> host pool */
  PA_SWAP_IN = 1   /* host pool -> device pools */
} pa_swap_dir;

/*
 * pa_swap_blocks - move whole blocks between the device pools and a host pool.
 *
 * When memory runs out, the server preempts: it evicts a sequence and later
 * recomputes or swaps its blocks back ("Paged Attention: Virtual Memory for
 * the KV Cache", section "What it does not fix"). This is the swap: for each
 * pair p, with (src, dst) = (block_pairs[2p], block_pairs[2p + 1]),
 *   PA_SWAP_OUT: host_k[dst] = k_cache[src]; host_v[dst] = v_cache[src]
 *   PA_SWAP_IN:  k_cache[dst] = host_k[src]; v_cache[dst] = host_v[src]
 * all heads of the block, bytes unchanged (the host pool keeps the cache's
 * in-block order; a block is num_kv_heads * block_size * head_dim elements).
 *
 *   host_k, host_v  page-locked host memory mapped into the device address
 *                   space (cudaHostAlloc / cudaHostRegister with the mapped
 *                   flag, or a pinned PyTorch tensor), host_num_blocks blocks
 *                   each, 16-byte aligned; PA_ERR_INVALID_ARG for memory the
 *                   device cannot address
 *   block_pairs     device int64 [num_pairs][2]; pairs with an index outside
 *                   its pool are skipped; every dst distinct
 *   direction       a pa_swap_dir
 * One kernel reads (or writes) the host pool directly over the host link; no
 * copy engine call per block. num_pairs == 0 is a no-op returning PA_OK.
 */
pa_status pa_swap_blocks(const pa_kv_cache* cache, void* host_k, void* host_v,
                         int32_t host_num_blocks, const int64_t* block_pairs,
                         int32_t num_pairs, int32_t direction, pa_stream_t stream);

/* Kernel choice for pa_decode (see pa_decode_options.path). */
typedef enum {
  PA_PATH_AUTO = 0,   /* tensor-core path when it applies, else CUDA cores */
  PA_PATH_SIMT = 1,   /* CUDA-core kernel for every supported shape */
  PA_PATH_TCGEN05 = 2 /* tensor-core kernel; PA_ERR_UNSUPPORTED if it cannot run */
} pa_decode_path;

typedef struct {
  /* Tokens per work item (context split). 0 = chosen on the device from the
     actual context lengths: pieces of up to one item stream's share of the
     whole batch (half a share when the batch has fewer (sequence, KV head)
     units than item streams; a multiple of 128, at least 256 and at least
     max_context_len / 64), listed longest first, with the ends of the
     sequences cut finer when the batch has too little short work to even out
     the finish. Otherwise a positive multiple of block_size with
     ceil(max_context_len / split_tokens) <= 256, every piece split_tokens
     long except each sequence's last. */
  int32_t split_tokens;
  int32_t path;        /* a pa_decode_path */
  /* 1 = read shared prefixes once per group of sequences (0 = off). Sequences
     forked from one another point at the same physical blocks for their
     common prefix ("Paged Attention: Virtual Memory for the KV Cache",
     "Sharing comes almost for free"). With this option the planning kernel
     compares each sequence's block table with the previous sequence's; runs
     of consecutive sequences sharing at least 256 tokens form groups of up
     to 16 query rows (16 / G sequences), and the whole pieces of their
     common prefix (pieces of at most 512 tokens unless split_tokens is set)
     are computed once for the group, reading each shared block once for all
     its members (on the tensor cores for 16-bit KV with head_dim 128 and G
     dividing 16, else on the CUDA cores), then merged with each member's own
     pieces. Results equal the per-sequence ones up to fp32 rounding. Applies
     to batches of 2 to 1024 sequences with G <= 8; elsewhere the option
     changes nothing. */
  int32_t share_prefixes;
} pa_decode_options;

/*
 * pa_decode_workspace_size - bytes of device workspace pa_decode needs for the
 * given shapes (status word and plan, work list, piece counts, the list of
 * sequences cut into pieces, a merge counter per (sequence, KV head), the
 * list of pieces shared by groups of sequences, one partial result per
 * (sequence, query head, piece)). split_tokens as in pa_decode_options.
 */
size_t pa_decode_workspace_size(int32_t num_seqs, int32_t num_q_heads,
                                int32_t head_dim, int32_t max_context_len,
                                int32_t block_size, int32_t split_tokens);

/*
 * pa_decode - paged single-query decode attention.
 *
 * For sequence i, query head h (0 <= h < num_q_heads) and KV head
 * kv = h / (num_q_heads / num_kv_heads) (consecutive query heads share a KV
 * head: grouped-query attention, "Paged Attention: Virtual Memory for the KV
 * Cache", "What it does not fix"):
 *   K_j = k_cache[bt[i][j / BS]][kv][j % BS][:],  V_j likewise,  j < L_i
 *   s_j = scale * <q[i][h], K_j>
 *   out[i][h] = sum_j exp(s_j - max s) V_j / sum_j exp(s_j - max s)
 * with bt = block_tables, L_i = context_lens[i]; L_i == 0 gives a zero row.
 * The sequence is read through its table in logical order, as though its
 * tokens sat back to back (glossary
 * "Paged attention", "What is Paged Attention?"). The pages never write the
 * formula; this is the plain scaled dot-product reading.
 *
 *   out           device fp32 [num_seqs, num_q_heads, head_dim]
 *   q             device [num_seqs, num_q_heads, head_dim], cache dtype
 *   block_tables  device int32 [num_seqs, bt_stride]
 *   context_lens  device int32 [num_seqs]; each <= max_context_len and
 *                 <= bt_stride * block_size
 *   max_context_len host-known upper bound of context_lens (sizes the split
 *                 grid and the workspace)
 *   opts          may be NULL (= split chosen on the device, path AUTO)
 *   workspace     device buffer of >= pa_decode_workspace_size(...) bytes,
 *                 16-byte aligned; owned by the caller, used by one call at a
 *                 time (two calls that overlap on the GPU must not share it).
 * Accumulation and softmax are fp32; the tensor-core path keeps the
 * probabilities at ~16 significant bits (two 16-bit terms).
 * PA_ERR_UNSUPPORTED also for more than 56,320 sequences in one call (the
 * planning kernel keeps the lengths in one CTA's shared memory), and for
 * num_seqs * num_q_heads of 2^31 or more (query rows are 32-bit copy
 * coordinates).
 * Enqueues two kernels: a planning kernel, then the decode kernel (three
 * with share_prefixes: the groups' shared pieces run as a decode launch of
 * their own before the decode kernel). The
 * planning kernel is launched with programmatic stream serialisation: it may
 * start while the kernel before it in the stream is finishing: it reads
 * context_lens and rewrites the workspace at once, then waits for that
 * kernel before it writes the zero rows of empty sequences into `out` and
 * completes. A kernel right before pa_decode that lets its dependents launch
 * early (griddepcontrol.launch_dependents) must by then have written
 * context_lens and be done with the workspace; it may still use `out`, q,
 * the tables and the pools.
 */
pa_status pa_decode(const pa_kv_cache* cache, float* out, const void* q,
                    const int32_t* block_tables, int32_t bt_stride,
                    const int32_t* context_lens, int32_t num_seqs,
                    int32_t num_q_heads, int32_t max_context_len, float scale,
                    const pa_decode_options* opts, void* workspace,
                    size_t workspace_bytes, pa_stream_t stream);

/*
 * pa_decode_noalloc - pa_decode for callers that cannot allocate device memory.
 *
 * The pages have no counterpart to this call. It exists for callers that
 * cannot obtain a workspace: a process that gives nearly all of HBM to its
 * KV-cache pool up front has no room left for a second allocation, and code on
 * a latency-critical path cannot afford cudaMalloc's implicit synchronisation.
 *
 * Arguments and result are those of pa_decode without the workspace. The
 * scratch is a fixed 32 MiB device array inside this library; every GPU that
 * loads the library holds it until the process exits. Shapes whose
 * pa_decode_workspace_size(...) exceeds 32 MiB are rejected with
 * PA_ERR_WORKSPACE_TOO_SMALL before anything is enqueued. The call allocates
 * nothing.
 *   - The first call on a device looks up the array's device address (with
 *     that device current) and keeps it for the life of the process; make
 *     that first call before any stream capture. cudaDeviceReset destroys the
 *     array with the context, so no call may follow a reset in the same
 *     process.
 *   - All calls share the one array and it keeps the last call's contents;
 *     each call re-initialises everything it reads, so nothing has to be
 *     cleared by the caller. Calls that overlap on the GPU (other streams, or
 *     other threads) race on the array and must not overlap.
 *   - The status word the kernels raise (see pa_decode_status) lives in the
 *     array too: read it with pa_decode_noalloc_status.
 */
pa_status pa_decode_noalloc(const pa_kv_cache* cache, float* out, const void* q,
                            const int32_t* block_tables, int32_t bt_stride,
                            const int32_t* context_lens, int32_t num_seqs,
                            int32_t num_q_heads, int32_t max_context_len,
                            float scale, const pa_decode_options* opts,
                            pa_stream_t stream);

/*
 * pa_decode_noalloc_status - pa_decode_status for pa_decode_noalloc: reads
 * back (synchronously, on `stream`) the status word that the last
 * pa_decode_noalloc on the current device left in the library's fixed
 * scratch, with the meanings given under pa_decode_status. The pages have no
 * counterpart to this call either; it exists because a pa_decode_noalloc
 * caller has no workspace pointer to hand to pa_decode_status. Returns
 * PA_ERR_CUDA if the scratch cannot be reached or the copy fails.
 */
pa_status pa_decode_noalloc_status(pa_stream_t stream);

/*
 * pa_decode_status - read back (synchronously, on `stream`) the device status
 * word the last pa_decode using `workspace` left: PA_OK;
 * PA_ERR_INVALID_ARG if a table entry was outside the pool (block 0 was read
 * in its place) or a length was negative or above max_context_len or its
 * table (that sequence's rows were written as zero); or
 * PA_ERR_DEVICE_TIMEOUT if one of its kernels stopped waiting on a barrier
 * after its time limit and returned early (its output is then invalid).
 * The word is cleared on every pa_decode. Returns PA_ERR_CUDA if the copy fails.
 */
pa_status pa_decode_status(const void* workspace, pa_stream_t stream);

/* Human-readable name of a status code (static string). */
const char* pa_status_string(pa_status status);

/* CUDA error string of the last PA_ERR_CUDA on this thread ("" if none). */
const char* pa_last_cuda_error(void);

/* Library version string. */
const char* pa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* PAGED_KV_CACHE_PA_H */
