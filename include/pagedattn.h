/*
 * pagedattn.h -- C ABI of the B200 (sm_100a) paged KV cache library.
 *
 * Decode-phase attention over a block-structured KV cache, as used by
 * nano-vLLM-style engines: a batch of sequences each brings one new query
 * token; each sequence's keys and values live in fixed-size physical blocks of
 * one shared pool and are reached through a per-sequence block table.
 *
 * Passages this interface follows (the pages print no kernel interface):
 *   - nano-vllm (ovshake) README, "Key Concepts Explained: PagedAttention":
 *     KV storage is a pool of fixed-size blocks handed to sequences on demand,
 *     in any physical order; each sequence keeps the list of its blocks.
 *   - same README, "Key Concepts Explained: KV Cache": a decode step computes
 *     K and V for the new token only and attends over everything cached.
 *   - same README, "X-Ray Mode", Steps 1-2: grouped-query attention (32 query
 *     heads share 8 KV heads) and scores Q K^T / sqrt(head_dim).
 *   - flex-nano-vllm README: paged attention with a page table serving
 *     Gemma 2 (the source of the tanh logit softcap and sliding window).
 *   - MinivLLM summary (sourcepulse), "How It Works": paging of the KV cache
 *     for decoding, blockwise exact attention.
 *
 * Conventions common to every call
 *   Cache layout ("HND"): k_cache and v_cache are row-major
 *     [num_blocks][num_kv_heads][block_size][head_dim] of dtype elements, so
 *     one (physical block, kv head) pair is one contiguous run of
 *     block_size * head_dim elements.  slot s names row (s % block_size) of
 *     block (s / block_size).
 *   Tensors q, out: [batch][num_q_heads][head_dim]; k, v (new rows):
 *     [num_tokens][num_kv_heads][head_dim]; block_tables:
 *     [batch][max_blocks_per_seq] int32 (entries past a sequence's last block
 *     are never read); context_lens: [batch] int32.
 *   context_lens[b] counts every cached token of sequence b, including the one
 *     appended this step (the query sits at position L-1).  L = 0 gives a zero
 *     output row.
 *   GQA: query head h reads kv head h / (num_q_heads / num_kv_heads).
 *   scale multiplies q.k; softcap c > 0 and finite replaces a scaled score x by
 *     c * tanh(x / c) (softcap <= 0 or +inf: no cap); window W > 0 keeps the
 *     last W positions [max(0, L-W), L) (W <= 0: no window).
 *   Supported: head_dim in {64, 128, 256}; block_size a power of two in
 *     [16, 256]; 1 <= num_q_heads / num_kv_heads <= 8 (integral);
 *     batch <= 65535; num_blocks * num_kv_heads * block_size < 2^31.
 *   Memory: every pointer is caller-owned DEVICE memory of the current device
 *     (q, caches, k, v, out, workspace 16-byte aligned; int32 arrays 4-byte;
 *     slot_mapping 8-byte).  The library allocates nothing and keeps no state
 *     beyond per-device constants and the device error word below.
 *   Streams: every call is asynchronous on `stream` (NULL = the legacy
 *     default stream); ordering follows stream order, so an append must be
 *     issued before the decode that reads it on the same stream.
 *   Errors: host checks run before anything is launched; a failed check
 *     returns an error status and launches nothing.  Kernels never trap: bad
 *     device-side values (a block id outside the pool, a slot outside the
 *     pool, a context longer than its table) skip the access and set a bit in
 *     the device error word, read back with pa_device_errors().
 */
#ifndef PAGEDATTN_H_
#define PAGEDATTN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

struct CUstream_st; /* cudaStream_t is `struct CUstream_st *` */
typedef struct CUstream_st* pa_stream_t;

typedef enum { PA_F32 = 0, PA_BF16 = 1 } pa_dtype_t;

typedef enum {
  PA_OK = 0,
  PA_ERR_INVALID = 1,     /* an argument failed a host check; nothing was launched */
  PA_ERR_UNSUPPORTED = 2, /* well-formed but outside what the kernels implement */
  PA_ERR_WORKSPACE = 3,   /* split-K workspace missing, misaligned or too small */
  PA_ERR_CUDA = 4         /* a CUDA runtime call or a launch failed */
} pa_status_t;

/* Which decode kernel runs.  AUTO picks the tensor-core kernel for bf16 and the
 * CUDA-core kernel for fp32.  MMA is bf16 only. */
typedef enum { PA_KERNEL_AUTO = 0, PA_KERNEL_CUDA_CORE = 1, PA_KERNEL_MMA = 2 } pa_kernel_t;

/* Decode schedules (see pa_decode_splitk), as reported by pa_last_decode_schedule. */
typedef enum {
  PA_SCHEDULE_NONE = 0,
  PA_SCHEDULE_SINGLE = 1,          /* one CTA per (sequence, kv head), no split */
  PA_SCHEDULE_GRID = 2,            /* one CTA per (partition, kv head, sequence), then the combine */
  PA_SCHEDULE_DYNAMIC = 3,         /* warp work queue, then the combine */
  PA_SCHEDULE_DYNAMIC_MERGED = 4   /* warp work queue, partitions merged in the same kernel */
} pa_schedule_t;

/* Bits of the device error word. */
enum {
  PA_DEVERR_SLOT = 1u,       /* write_kv: slot >= num_blocks * block_size (row skipped) */
  PA_DEVERR_BLOCK = 2u,      /* decode: block id outside [0, num_blocks) (tile skipped) */
  PA_DEVERR_CONTEXT = 4u,    /* decode: context_lens[b] < 0 or > max_blocks_per_seq * block_size,
                                or > max_context_len in split-K (length clamped) */
  PA_DEVERR_TIMEOUT = 8u,    /* a bounded wait on a tile load gave up (output row not written) */
  PA_DEVERR_LAYOUT = 16u     /* prefill: shared memory was not 1024-byte aligned (tile not computed) */
};

/*
 * pa_write_kv -- append one step's new key/value rows into the paged cache.
 *   For every i < num_tokens with slot_mapping[i] >= 0 and every kv head h:
 *     k_cache[s / bs][h][s % bs][:] = k[i][h][:]   (and the same for v)
 *   The copy is bit-exact.  slot_mapping[i] < 0 marks a padding token (skipped).
 *   A slot >= num_blocks * block_size sets PA_DEVERR_SLOT and is skipped.
 *   Two tokens with the same slot in one call: which one lands is undefined.
 *   Passage: nano-vllm README, "Key Concepts Explained: KV Cache" (only the new
 *   token's K and V are computed; the rest are reused from the cache).
 *   Returns PA_ERR_INVALID for null/misaligned pointers or bad sizes.
 */
pa_status_t pa_write_kv(const void* k, const void* v, const int64_t* slot_mapping, int32_t num_tokens,
                        void* k_cache, void* v_cache, int32_t num_blocks, int32_t block_size,
                        int32_t num_kv_heads, int32_t head_dim, pa_dtype_t dtype, pa_stream_t stream);

/*
 * pa_decode -- paged decode attention, one CTA per (sequence, kv head).
 *   out[b][h][:] = sum_t softmax_t(x) V[b][g][t][:],  t in [s0, L),
 *   x_t = scale * q[b][h] . K[b][g][t]  (then the softcap), g = h / G,
 *   where K[b][g][t] is row t % bs of block block_tables[b][t / bs].
 *   Accumulation and the softmax state are fp32; out has the input dtype
 *   (bf16 rounded to nearest even).  Needs no workspace.
 *   Passages: see the file header (PagedAttention, KV Cache, X-Ray Mode).
 */
pa_status_t pa_decode(const void* q, const void* k_cache, const void* v_cache, const int32_t* block_tables,
                      const int32_t* context_lens, int32_t batch, int32_t num_q_heads, int32_t num_kv_heads,
                      int32_t head_dim, int32_t block_size, int32_t max_blocks_per_seq, int32_t num_blocks,
                      float scale, float softcap, int32_t window, void* out, pa_dtype_t dtype,
                      pa_kernel_t kernel, pa_stream_t stream);

/*
 * Split-K (flash-decoding) variant for long contexts and small batches.
 *   Each sequence's attended range is cut at multiples of partition_tokens;
 *   one CTA per (partition, kv head, sequence) writes its partial softmax state
 *   (running max m, sum l, unnormalised output o, all fp32) to the workspace,
 *   and a second kernel merges the partials with a log-sum-exp combine:
 *     M = max_p m_p,  out = sum_p e^(m_p - M) o_p / sum_p e^(m_p - M) l_p.
 *   A sequence whose range falls in one partition is written directly by that
 *   partition's CTA; its result is then bit-identical to pa_decode's.
 *   The combine kernel is launched as a programmatic dependent of the first
 *   (its launch overlaps the first kernel's tail; it reads nothing before the
 *   first kernel has completed).
 *   partition_tokens: a multiple of 64, or 0 to let the library choose (see
 *   pa_decode_splitk_partition).  max_context_len: an upper bound on every
 *   context_lens[b] (a larger length sets PA_DEVERR_CONTEXT and is clamped);
 *   it sizes the grid and the workspace.
 *   Schedules: partition_tokens > 0 launches one CTA per (partition, kv head,
 *   sequence).  partition_tokens == 0 lets the library choose the partition
 *   size and, on the tensor-core path (bf16) with batch <= 2048 and
 *   batch * num_kv_heads <= 65534, runs the
 *   dynamic schedule: one persistent kernel whose warps claim (sequence, kv
 *   head, partition) items from a counter kept in the workspace, so that SMs
 *   that stream faster take more of the work; the last partial of each
 *   (sequence, kv head) to arrive merges the others in the same kernel, so no
 *   combine kernel runs.
 *   workspace: device memory of at least pa_decode_splitk_workspace_size()
 *   bytes, 16-byte aligned, zero-filled before its first use.  It starts with
 *   a fixed 256 KiB counter region (the dynamic schedule's counters, which
 *   return to zero at the end of every call), followed by the partials
 *   (scratch within a call).  A workspace sized for the largest call serves
 *   calls of any smaller shape and either schedule in any order without being
 *   zeroed again.  After a call that failed or raised PA_DEVERR_TIMEOUT, zero
 *   it again.  Calls that share a workspace must be ordered on one stream.
 *   Returns PA_ERR_WORKSPACE when the workspace is null, misaligned or small.
 */
int32_t pa_decode_splitk_partition(int32_t batch, int32_t num_kv_heads, int32_t max_context_len,
                                   int32_t partition_tokens);
size_t pa_decode_splitk_workspace_size(int32_t batch, int32_t num_q_heads, int32_t head_dim,
                                       int32_t max_context_len, int32_t partition_tokens,
                                       int32_t num_kv_heads);
pa_status_t pa_decode_splitk(const void* q, const void* k_cache, const void* v_cache, const int32_t* block_tables,
                             const int32_t* context_lens, int32_t batch, int32_t num_q_heads,
                             int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                             int32_t max_blocks_per_seq, int32_t num_blocks, float scale, float softcap,
                             int32_t window, void* out, pa_dtype_t dtype, int32_t partition_tokens,
                             int32_t max_context_len, void* workspace, size_t workspace_bytes,
                             pa_kernel_t kernel, pa_stream_t stream);

/*
 * pa_decode_step -- one decode step: append the step's new key/value rows and
 * attend, in one pass over the cache.
 *   Equivalent to pa_write_kv(k_new, v_new, slots) followed by the decode, where
 *   slots[b] is the slot of position L-1 of sequence b, i.e.
 *   block_tables[b][(L-1)/bs] * bs + (L-1) % bs with L = context_lens[b]
 *   (nothing is appended for L == 0).  k_new, v_new: [batch][num_kv_heads]
 *   [head_dim], device memory, 16-byte aligned.  The cache must not be read by
 *   other work while the call runs; the block receiving position L-1 must not be
 *   shared with another sequence (prefix-shared blocks are full and never the
 *   one being appended to).
 *   The attention uses the new rows from on-chip memory, and the CTA that
 *   serves position L-1 of (sequence, kv head) writes them to the cache, so no
 *   separate append kernel runs.  The outputs and the cache contents equal those
 *   of pa_write_kv followed by pa_decode / pa_decode_splitk bit for bit.
 *   partition_tokens < 0: one CTA per (sequence, kv head), like pa_decode (the
 *   workspace may be NULL and max_context_len is ignored).  partition_tokens >= 0:
 *   split-K exactly as pa_decode_splitk (0 = library's choice).
 *   Passage: nano-vllm README, "Key Concepts Explained: KV Cache" (each decode
 *   step processes only the new token and attends over the cache).
 */
pa_status_t pa_decode_step(const void* q, const void* k_new, const void* v_new, void* k_cache, void* v_cache,
                           const int32_t* block_tables, const int32_t* context_lens, int32_t batch,
                           int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                           int32_t max_blocks_per_seq, int32_t num_blocks, float scale, float softcap,
                           int32_t window, void* out, pa_dtype_t dtype, int32_t partition_tokens,
                           int32_t max_context_len, void* workspace, size_t workspace_bytes, pa_kernel_t kernel,
                           pa_stream_t stream);

/*
 * pa_decode_multi -- attention for several new query tokens per sequence
 * (speculative-decoding verify, one chunk of a chunked prefill).
 *   q: [batch][q_len][num_q_heads][head_dim] bf16; out: the same shape.  The
 *   q_len new tokens' keys and values must already be in the cache (append
 *   them with pa_write_kv first) at positions L-q_len .. L-1, L =
 *   context_lens[b].  Query token j sits at position p_j = L - q_len + j and
 *   attends causally: positions t with s0_j <= t <= p_j, where s0_j = p_j + 1
 *   - window when window > 0 and p_j + 1 > window, else 0; scores, softcap
 *   and softmax as pa_decode.  A token with p_j < 0 (L < q_len) gets a zero
 *   row; L = 0 gives zero rows.
 *   bf16 only (PA_ERR_UNSUPPORTED for fp32); q_len * (num_q_heads /
 *   num_kv_heads) <= 64 (PA_ERR_UNSUPPORTED above).
 *   partition_tokens < 0: one CTA per (sequence, kv head), no workspace
 *   (workspace may be NULL; max_context_len is ignored).  partition_tokens >= 0:
 *   split-K (0 = library's choice) with a workspace of
 *   pa_decode_multi_workspace_size() bytes under the same contract as
 *   pa_decode_splitk's, and a combine kernel for sequences whose range spans
 *   several partitions.  With at most 16 query rows per kv head (q_len *
 *   num_q_heads / num_kv_heads; 32 at head_dim 64) the rows run on
 *   pa_decode_splitk's warp-per-item schedule, one warp per (sequence, kv
 *   head, partition); above that, on one CTA per (partition, kv head,
 *   sequence).
 *   Passages: nano-vllm (ovshake) README, "Features" (chunked prefill,
 *   speculative decoding) and the speculative-decoding command line
 *   (--num-speculative-tokens); causal attention over the cache as in "Key
 *   Concepts Explained: KV Cache".
 */
pa_status_t pa_decode_multi(const void* q, const void* k_cache, const void* v_cache, const int32_t* block_tables,
                            const int32_t* context_lens, int32_t batch, int32_t q_len, int32_t num_q_heads,
                            int32_t num_kv_heads, int32_t head_dim, int32_t block_size, int32_t max_blocks_per_seq,
                            int32_t num_blocks, float scale, float softcap, int32_t window, void* out,
                            pa_dtype_t dtype, int32_t partition_tokens, int32_t max_context_len, void* workspace,
                            size_t workspace_bytes, pa_stream_t stream);
size_t pa_decode_multi_workspace_size(int32_t batch, int32_t q_len, int32_t num_q_heads, int32_t head_dim,
                                      int32_t max_context_len, int32_t partition_tokens, int32_t num_kv_heads);

/*
 * pa_prefill -- paged prefill: append a batch of prompts' (or prompt chunks')
 * key/value rows and attend them causally over the paged cache.
 *   Sequence b's new tokens are rows [cu_q_lens[b], cu_q_lens[b+1]) of q
 *   ([total_q][num_q_heads][head_dim]), k_new, v_new ([total_q][num_kv_heads]
 *   [head_dim]), slot_mapping ([total_q] int64) and out (like q): T_b tokens,
 *   the last T_b positions of the context, L = context_lens[b] (which counts
 *   them).  cu_q_lens: [batch + 1] int32 device array, non-decreasing, with
 *   cu_q_lens[batch] <= total_q and every T_b <= max_q_len (else
 *   PA_DEVERR_CONTEXT and the sequence's rows are not written).
 *   First the rows are appended exactly as pa_write_kv(k_new, v_new,
 *   slot_mapping, total_q) does; pass k_new = v_new = NULL to skip the append
 *   when the rows are already in the cache.  Then token j of sequence b, at
 *   position p = L - T_b + j, attends positions [s0, p] as in pa_decode_multi
 *   (causal, window, softcap).  A chunk of a chunked prefill is the same call
 *   with the earlier chunks already in the cache.
 *   bf16 only.  One launch for the append and one for the attention, whose
 *   CTAs each take 128 / G query tokens of one sequence and one kv head
 *   (max_q_len / (128 / G) <= 65535, else PA_ERR_UNSUPPORTED), each
 *   sequence's last tokens (the most keys under the causal mask) first; no
 *   workspace.
 *   Passages: nano-vllm (ovshake) README, "Key Concepts Explained: KV Cache"
 *   (prefill processes the prompt and stores its keys and values) and
 *   "Features" (chunked prefill); MinivLLM (the pages' second project) times
 *   prefilling and decoding separately.
 */
pa_status_t pa_prefill(const void* q, const void* k_new, const void* v_new, const int64_t* slot_mapping,
                       const int32_t* cu_q_lens, int32_t total_q, int32_t max_q_len, void* k_cache, void* v_cache,
                       const int32_t* block_tables, const int32_t* context_lens, int32_t batch, int32_t num_q_heads,
                       int32_t num_kv_heads, int32_t head_dim, int32_t block_size, int32_t max_blocks_per_seq,
                       int32_t num_blocks, float scale, float softcap, int32_t window, void* out, pa_dtype_t dtype,
                       pa_stream_t stream);

/*
 * pa_decode_cascade -- split-K decode that reads a shared prefix once.
 *   Sequences 0 .. n_sharers-1 of the batch share their first prefix_len
 *   positions: the first prefix_len / block_size entries of their block
 *   tables are the same physical blocks, holding valid rows (prefix caching
 *   shares full blocks).  The result equals pa_decode_splitk's, within the
 *   same tolerance; only the order of the additions differs.
 *   Three launches: (1) the prefix pass loads each prefix block once per kv
 *   head and attends it for every sharer (64 / G sharers x G query heads per
 *   CTA, on the multi-query kernel), writing split-K partials; (2) the
 *   split-K decode attends every sequence's own range (sharers from position
 *   prefix_len on); (3) the log-sum-exp combine merges both.  A sharer whose
 *   table differs from sequence 0's inside the prefix raises PA_DEVERR_BLOCK
 *   (its prefix rows are then sequence 0's).
 *   prefix_len: a multiple of 64 and of block_size, <= max_context_len and
 *   <= max_blocks_per_seq * block_size (else PA_ERR_INVALID).
 *   partition_tokens: 0 lets the library choose (halved until it divides
 *   prefix_len), else a multiple of 64 that divides prefix_len.  The workspace
 *   is pa_decode_cascade_workspace_size() bytes under pa_decode_splitk's
 *   contract.  n_sharers = 0 or prefix_len = 0 runs pa_decode_splitk.  bf16.
 *   Passages: nano-vllm (ovshake) README, "Features" ("Prefix Caching: share
 *   KV cache blocks for common prefixes") and "PagedAttention" (sequences
 *   reach shared blocks through their tables).
 */
pa_status_t pa_decode_cascade(const void* q, const void* k_cache, const void* v_cache, const int32_t* block_tables,
                              const int32_t* context_lens, int32_t batch, int32_t num_q_heads, int32_t num_kv_heads,
                              int32_t head_dim, int32_t block_size, int32_t max_blocks_per_seq, int32_t num_blocks,
                              float scale, float softcap, int32_t window, void* out, pa_dtype_t dtype,
                              int32_t n_sharers, int32_t prefix_len, int32_t partition_tokens,
                              int32_t max_context_len, void* workspace, size_t workspace_bytes, pa_stream_t stream);
size_t pa_decode_cascade_workspace_size(int32_t batch, int32_t num_q_heads, int32_t head_dim,
                                        int32_t max_context_len, int32_t prefix_len, int32_t partition_tokens,
                                        int32_t num_kv_heads);

/*
 * pa_decode_splitk_noalloc -- pa_decode_splitk for callers that cannot allocate
 * device memory.
 *   The pages describe no such call; it exists for callers that must not call
 *   cudaMalloc (or any allocating routine) on their path: code running inside
 *   a CUDA stream capture that forbids allocation, real-time serving loops that
 *   cannot afford an allocation's synchronisation, and hosts whose memory is
 *   handed out by a foreign allocator the library cannot reach.  Such a caller
 *   passes the same inputs and output as to pa_decode_splitk but no workspace:
 *   the split-K scratch is a fixed array of PA_NOALLOC_SCRATCH_BYTES in the
 *   library's own device memory (reserved on every GPU that loads the library,
 *   for the life of the process).
 *   Returns PA_ERR_WORKSPACE when the call would need more scratch than that
 *   (pa_decode_splitk_workspace_size() > PA_NOALLOC_SCRATCH_BYTES); such calls
 *   must use pa_decode_splitk with a workspace of their own.
 *   The first call on a device looks up the array's device address (no
 *   allocation; it may load the library's module on that device): make that
 *   first call before any stream capture.  The address is looked up again
 *   whenever the device's context has changed since (after a
 *   cudaDeviceReset), so the call stays valid across a reset; the first call
 *   after a reset is again a first call.  Any device ordinal is served.
 *   Every call uses the same array, and it keeps what the last call left in
 *   it: when the dynamic schedule runs (partition_tokens == 0 on the
 *   tensor-core path), the call first clears the part of the array that must
 *   start at zero (the schedule's counters, at its start) with an
 *   asynchronous memset on `stream`; a call rejected by a host check touches
 *   neither the device nor the array.  Calls whose executions overlap on the
 *   GPU (different streams, or different host threads without ordering) race
 *   on the array and give wrong results; order them.
 *   It allocates nothing: no cudaMalloc, no cudaFree, no allocating library call.
 */
#define PA_NOALLOC_SCRATCH_BYTES (16u << 20) /* 16 MiB */
pa_status_t pa_decode_splitk_noalloc(const void* q, const void* k_cache, const void* v_cache,
                                     const int32_t* block_tables, const int32_t* context_lens, int32_t batch,
                                     int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                                     int32_t block_size, int32_t max_blocks_per_seq, int32_t num_blocks,
                                     float scale, float softcap, int32_t window, void* out, pa_dtype_t dtype,
                                     int32_t partition_tokens, int32_t max_context_len, pa_kernel_t kernel,
                                     pa_stream_t stream);

/*
 * pa_device_errors -- read (and with clear != 0, reset) the device error word
 * of the current device.  Synchronises with the device.  *bits receives the
 * OR of every PA_DEVERR_* raised since the last clear.
 */
pa_status_t pa_device_errors(uint32_t* bits, int32_t clear);

/*
 * pa_check_bounded_wait -- diagnostic: launch one CTA that waits on an
 * mbarrier nothing ever arrives on, with the bounded wait every kernel of this
 * library uses for its TMA and MMA completions.  The wait gives up after
 * limit_ns nanoseconds of %globaltimer (0 < limit_ns <= 1e9, else
 * PA_ERR_INVALID) and raises PA_DEVERR_TIMEOUT in the device error word; the
 * kernel then returns and the context stays usable.  It shows on a GPU that
 * a wait that never completes ends in an error status instead of a hang.
 * Asynchronous on stream; read the result with pa_device_errors().
 */
pa_status_t pa_check_bounded_wait(uint64_t limit_ns, pa_stream_t stream);

/* Static description of a status code. */
const char* pa_error_string(pa_status_t status);

/* Number of kernels the last successful call on this host thread launched
 * (0 after a failed call).  For accounting in benchmarks. */
int32_t pa_last_launch_count(void);

/* The schedule the last decode call (pa_decode, pa_decode_splitk,
 * pa_decode_splitk_noalloc, pa_decode_step) on this host thread ran: one of
 * pa_schedule_t, PA_SCHEDULE_NONE after a failed call or a call that launched
 * nothing.  For tests and benchmarks that report which path ran. */
int32_t pa_last_decode_schedule(void);

#ifdef __cplusplus
}
#endif

#endif /* PAGEDATTN_H_ */
