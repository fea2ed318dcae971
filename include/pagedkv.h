/*
 * pagedkv -- paged KV cache decode on B200 (sm_100a): C ABI.
 *
 * The KV cache of every running sequence lives in fixed-size blocks of
 * `block_size` tokens drawn from one shared physical pool; a per-sequence block
 * table maps logical block j (tokens j*block_size .. (j+1)*block_size-1) to a
 * physical block.  Sources (web pages, cited by site, title and section):
 *   [E]  openeuler.csdn.net, PagedAttention explainer: 2.1-2.2 decode and the
 *        KV cache, 4.1 fixed-size blocks, 4.2 block table (logical ->
 *        physical), 4.3 on-demand growth, 6.1 shared prefix, 6.2
 *        copy-on-write.
 *   [B]  agent.csdn.net, PagedAttention blog: 2.1 blocks of 16 tokens, only the
 *        last block partly filled; 2.2 copy-on-write for parallel samples and
 *        beams; 3.1 block-manager sketch (allocate a free block on demand);
 *        4.2 bandwidth decides the fastest precision.
 *   [T]  aiknowledge.cn, "2.2 PagedAttention 与 KV Cache 分页管理": 2.2.2 free
 *        pool, blocks freed on finish or preemption; 2.2.3 worked example
 *        (35 tokens -> physical blocks 7, 3, 9) and prefix sharing; 2.2.4 a
 *        kernel fused over non-contiguous blocks; 2.2.8 byte-identical
 *        prefixes reused; 2.2.13 pool monitoring.
 *
 * Conventions for every call
 *   - Device pointers are caller-owned device memory, 16-byte aligned; the
 *     library never allocates device memory (the split-K workspace is passed
 *     in; query its size first).
 *   - Sizes are trusted: the library cannot see a buffer's extent, so every
 *     buffer must hold at least what its size arguments describe (a table
 *     row and a length per sequence, a slot per new token, q-shaped output);
 *     a shorter one is read or written past its end.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Device calls are asynchronous on that stream.
 *   - Host-side validation happens before any launch; a rejected call returns
 *     PKV_ERR_INVALID / PKV_ERR_UNSUPPORTED and launches nothing.  A failed
 *     launch returns PKV_ERR_CUDA.  pkv_last_error() gives a message.
 *   - Kernels check every index they read from device memory (block ids,
 *     slots, context lengths).  A bad one is not dereferenced: the kernel
 *     records a bit in a device error word and carries on with a safe value,
 *     so the output is then meaningless but no fault occurs.  Read and clear
 *     the word with pkv_device_error().
 *   - No C++ exception crosses this boundary.
 *
 * Pool layout (K and V pools alike, one array each):
 *     pool[num_blocks][num_kv_heads][block_size][head_dim], row-major,
 * so the `block_size x head_dim` tile of one (block, kv head) is contiguous.
 * Element types: PKV_F32, PKV_BF16, PKV_F16; q, new K/V, pools and the output
 * of one call share one type, except in the _fp8 calls (FP8 E4M3 pools with
 * 16-bit q and output).
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
    PKV_ERR_INVALID = 1,        /* bad argument; nothing was done */
    PKV_ERR_NO_FREE_BLOCK = 2,  /* allocator: pool exhausted; nothing changed */
    PKV_ERR_CUDA = 3,           /* a CUDA runtime call or launch failed */
    PKV_ERR_UNSUPPORTED = 4,    /* valid but not built (e.g. head_dim 96) */
    PKV_ERR_DEVICE_CHECK = 5    /* pkv_device_error found a recorded bad index */
} pkv_status;

typedef enum { PKV_F32 = 0, PKV_BF16 = 1, PKV_F16 = 2, PKV_FP8_E4M3 = 3 /* pools of the _fp8 calls only */ } pkv_dtype;

/* Bits of the device error word. */
#define PKV_DEVERR_BLOCK_ID   1u  /* block id outside [0, num_blocks) */
#define PKV_DEVERR_SLOT       2u  /* slot outside [0, num_blocks*block_size) */
#define PKV_DEVERR_CONTEXT    4u  /* context length < 0 or > max_blocks_per_seq*block_size */
#define PKV_DEVERR_TIMEOUT    8u  /* a bounded wait on an async copy gave up */
#define PKV_DEVERR_GROUP     16u  /* a shared-prefix group description does not hold: more members than
                                     max_group_size, a shared run over max_shared_len, or a member whose
                                     leading blocks are not its group's */
#define PKV_DEVERR_SPLIT     32u  /* a split-K counter word changed under a call in a way its own
                                     partitions cannot explain (the workspace was in use by another
                                     call at the same time); that row's output is not written */

/* ------------------------------------------------------------------ device */

/*
 * pkv_kv_append -- write each new token's K and V into its slot.
 * [E] 2.2 (each step caches one new K/V), [T] 2.2.3 (the token lands in the
 * sequence's last block), [E] 4.3 (growth by whole blocks).
 *   k_new, v_new   [T][num_kv_heads][head_dim]
 *   k_pool, v_pool [num_blocks][num_kv_heads][block_size][head_dim]
 *   slot_mapping   int64 [T]; token i goes to block slot/block_size at offset
 *                  slot%block_size.  slot < 0 = skip the token.  Slots must be
 *                  distinct (duplicates: unspecified which token wins).
 * Bit-exact byte copy.  Supported head_dim*elem_size multiple of 16 bytes.
 */
pkv_status pkv_kv_append(const void* k_new, const void* v_new, void* k_pool, void* v_pool,
                         const int64_t* slot_mapping, int num_tokens, int num_blocks,
                         int num_kv_heads, int head_dim, int block_size, pkv_dtype dtype,
                         void* stream);

/*
 * Bytes of split-K workspace pkv_paged_attention_decode needs.
 *   max_context_len  upper bound on any context length of the call; the decode
 *                    call uses max_blocks_per_seq*block_size as that bound.
 *   partition_size   as in the decode call (0 = library's choice; the size
 *                    returned then covers whatever the library picks).
 * Returns 0 when no workspace is needed (every context fits one partition),
 * and SIZE_MAX when the size does not fit in size_t (such a call cannot run).
 * Layout, for R = num_seqs*num_q_heads rows and N partitions: R*N*head_dim
 * floats of partial outputs, R*N*2 floats of (max, sum) pairs, then, from the
 * next 256-byte boundary, R 8-byte split counters, with which a decode
 * kernel merges a row's partials itself once the row's last partition has
 * finished (no reduce kernel).  A counter word holds a 48-bit stamp of the
 * call that wrote it, so stale contents are ignored and the workspace needs
 * no initialisation; one call at a time per workspace.
 */
size_t pkv_attention_workspace_bytes(int num_seqs, int num_q_heads, int head_dim,
                                     int max_context_len, int partition_size);

/* The partition size (tokens) the decode call will use for these arguments. */
int pkv_attention_partition_size(int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                                 int max_context_len, int partition_size);

/*
 * pkv_paged_attention_decode -- one query token per sequence attends to its
 * cached tokens, read block by block through its block table
 * ([E] 4.2: the kernel reads the KV cache block by block through the block
 *  table; [T] 2.2.4 fused over non-contiguous blocks).  For sequence s, query head h:
 *     g   = h / (num_q_heads / num_kv_heads)   (grouped-query attention)
 *     x_t = scale * q[s,h,:] . K[slot(s,t), g, :],  t < context_lens[s]
 *     out[s,h,:] = sum_t softmax(x)_t V[slot(s,t), g, :]
 *     slot(s,t) = block_tables[s][t / block_size] * block_size + t % block_size
 * No mask; context_lens[s] = 0 gives zeros.  Accumulation is fp32 (online
 * softmax); the result is rounded once to the element type.
 *   out, q          [num_seqs][num_q_heads][head_dim]
 *   block_tables    int32 [num_seqs][max_blocks_per_seq]; entries past a
 *                   sequence's last block are never read.
 *   context_lens    int32 [num_seqs], 0 <= len <= max_blocks_per_seq*block_size
 *   scale           0 -> 1/sqrt(head_dim)
 *   partition_size  0 -> library's choice; > 0 (multiple of 16) splits every
 *                   context into partitions of that many tokens that run in
 *                   parallel, then a reduce kernel merges them (the MHA
 *                   kernels merge their own when there are at most 32
 *                   partitions of at least 512 tokens, without groups).
 *                   For at most 256 sequences and 1024 sequences x
 *                   partitions per call, the MHA kernels start partitions
 *                   longest first: every sequence's full partitions, then
 *                   its short last ones by decreasing length (the same
 *                   partitions, in another order).
 *   workspace       >= pkv_attention_workspace_bytes(...) bytes of device
 *                   memory, 256-byte aligned; contents need no initialisation.
 * Supported: head_dim 64 or 128; block_size 16, 32, 64, 128 or 256;
 * num_blocks*num_kv_heads*block_size < 2^31; at most 65535 sequences, query
 * heads and partitions per call.  16-bit types with a query group
 * of 2..16 heads run on tensor cores; other cases on CUDA cores.
 * Deterministic: the same inputs give bit-identical outputs.
 */
pkv_status pkv_paged_attention_decode(void* out, const void* q, const void* k_pool, const void* v_pool,
                                      const int32_t* block_tables, int max_blocks_per_seq,
                                      const int32_t* context_lens, int num_seqs, int num_q_heads,
                                      int num_kv_heads, int head_dim, int block_size, int num_blocks,
                                      float scale, int partition_size, void* workspace,
                                      size_t workspace_bytes, pkv_dtype dtype, void* stream);

/*
 * pkv_paged_attention_decode_shared -- the same decode attention for a batch
 * in which runs of consecutive sequences share their first tokens in the same
 * physical blocks (one system prompt stored once and referenced by every
 * sequence: [E] 6.1, [T] 2.2.3).  The result equals pkv_paged_attention_decode
 * on the same inputs (up to fp32 rounding order).  The shared tokens are
 * attended once per group by a prefix pass in which every warp multiplies 16
 * queries of the group (sequence x head pairs) by each shared K/V tile on
 * tensor cores, so a shared tile is read once per 16 queries instead of once
 * per query; each sequence's own tokens go through the usual split-K pass and
 * one reduce merges both.
 *   group_first   device int32 [num_groups + 1], non-decreasing, within
 *                 [0, num_seqs]: group g is sequences group_first[g] ..
 *                 group_first[g+1]-1.  Sequences outside every group are
 *                 handled as in pkv_paged_attention_decode.
 *   group_shared  device int32 [num_groups]: number of leading tokens the
 *                 members of group g share, a multiple of block_size, at most
 *                 every member's context length.  A value breaking these
 *                 rules is recorded (PKV_DEVERR_CONTEXT) and the members it
 *                 breaks them for are handled as non-members.
 *                 The prefix pass reads the first group_shared[g]/block_size
 *                 block-table entries of the group's first sequence; only
 *                 members whose own first entries are the same take its
 *                 result ([E] 6.1, [T] 2.2.8: only identical prefixes are
 *                 shared).  The call compares them on the device, once
 *                 per sequence, before its attention kernels run; a member
 *                 whose entries differ is recorded (PKV_DEVERR_GROUP) and
 *                 handled as a non-member.
 *   max_group_size  host bound on members per group (it sizes the prefix
 *                 pass); members past it are recorded (PKV_DEVERR_GROUP)
 *                 and handled as non-members.
 *   max_shared_len  host bound on every group_shared[g] (it sizes the prefix
 *                 pass); a larger group_shared is recorded as
 *                 PKV_DEVERR_GROUP and its members handled as non-members.
 * A non-member attends to its whole context through its own table, so the
 * result equals pkv_paged_attention_decode's whatever the group description
 * says; only the speed depends on it.
 *   workspace     >= pkv_attention_shared_workspace_bytes(...) bytes.
 * 16-bit element types only (PKV_ERR_UNSUPPORTED for fp32).
 */
pkv_status pkv_paged_attention_decode_shared(void* out, const void* q, const void* k_pool, const void* v_pool,
                                             const int32_t* block_tables, int max_blocks_per_seq,
                                             const int32_t* context_lens, int num_seqs, int num_q_heads,
                                             int num_kv_heads, int head_dim, int block_size, int num_blocks,
                                             float scale, int partition_size, const int32_t* group_first,
                                             const int32_t* group_shared, int num_groups, int max_group_size,
                                             int max_shared_len, void* workspace, size_t workspace_bytes,
                                             pkv_dtype dtype, void* stream);

/* Workspace bytes for pkv_paged_attention_decode_shared (arguments as in
 * pkv_attention_workspace_bytes; never 0 for num_seqs > 0): the split-K
 * partials with one extra slot per row, then 8 bytes per sequence in which
 * the call records, once, whether the sequence takes its group's prefix
 * result. */
size_t pkv_attention_shared_workspace_bytes(int num_seqs, int num_q_heads, int head_dim, int max_context_len,
                                            int partition_size);

/*
 * Host helper: find runs of consecutive sequences whose block tables start
 * with the same physical blocks (what pkv_paged_attention_decode_shared
 * needs).  block_tables / context_lens are HOST arrays ([n][max_blocks],
 * [n]).  A run of at least min_group_size sequences whose tables agree on
 * their first k >= 1 entries, all full blocks of every member, becomes a
 * group sharing k*block_size tokens (the greedy run from its first member;
 * k is the smallest agreement inside the run).  The output partitions
 * 0..n-1 into runs -- the groups and the gaps between them, the latter with
 * group_shared = 0 -- in the format pkv_paged_attention_decode_shared takes:
 * group_first[0..n_groups] (group_first[n_groups] = n) and
 * group_shared[0..n_groups-1].  max_groups must be >= n (group_first then
 * needs n + 1 entries).
 */
pkv_status pkv_find_shared_prefix_groups(const int32_t* block_tables, const int32_t* context_lens, int n,
                                         int max_blocks, int block_size, int min_group_size,
                                         int32_t* group_first, int32_t* group_shared, int max_groups,
                                         int* n_groups);

/*
 * pkv_paged_attention_chunk -- causal attention for a chunk of new tokens per
 * sequence (speculative verification of draft tokens, or a short chunk of a
 * prompt), read through the block tables like decode.  Sequence s owns query
 * rows query_start[s] .. query_start[s+1]-1 (n_s rows), which are the last
 * n_s of its context_lens[s] cached tokens (their K/V already appended);
 * row i sits at position context_lens[s] - n_s + i and attends to tokens
 * 0 .. context_lens[s] - n_s + i: itself and everything before it
 * ([E] 2.1-2.2: each new token attends to all earlier ones).  n_s = 1 is
 * decode.
 *   out, q        [num_tokens][num_q_heads][head_dim]
 *   query_start   device int32 [num_seqs + 1], non-decreasing, within
 *                 [0, num_tokens]; n_s <= context_lens[s] and <= max_query_len
 *                 (a violation is recorded as PKV_DEVERR_CONTEXT and that
 *                 sequence's rows are left untouched).
 *   max_query_len host bound on n_s.
 *   workspace     >= pkv_attention_chunk_workspace_bytes(...) bytes.
 * 16-bit element types, query groups of 1..16 heads (tensor cores: the 16
 * rows of an MMA are (new token, head) pairs).
 */
pkv_status pkv_paged_attention_chunk(void* out, const void* q, const void* k_pool, const void* v_pool,
                                     const int32_t* block_tables, int max_blocks_per_seq,
                                     const int32_t* context_lens, const int32_t* query_start, int num_seqs,
                                     int num_tokens, int max_query_len, int num_q_heads, int num_kv_heads,
                                     int head_dim, int block_size, int num_blocks, float scale,
                                     int partition_size, void* workspace, size_t workspace_bytes,
                                     pkv_dtype dtype, void* stream);

/* Workspace bytes for pkv_paged_attention_chunk (0 if no context needs splitting). */
size_t pkv_attention_chunk_workspace_bytes(int num_tokens, int num_q_heads, int head_dim, int max_context_len,
                                           int partition_size);

/*
 * Quantized KV pools: FP8 E4M3 codes (1 byte per element, same layout as the
 * other pools).  The pages only say that bandwidth decides which precision
 * serves fastest ([B] 4.2); the scheme here: one scale per pool, a stored
 * code c stands for e4m3(c) * k_scale (K) or * v_scale (V), halving the bytes
 * decode attention streams.  E4M3: sign, 4 exponent bits (bias 7), 3 mantissa
 * bits, largest finite 448, no infinities.
 *
 * pkv_kv_append_fp8 -- as pkv_kv_append, but the new K/V (src_dtype: f32,
 * bf16 or f16) are quantized: code = e4m3(x * (1/scale)), the inverse scale
 * rounded to fp32 once, the product computed in fp32, rounded to nearest
 * (ties to even) and saturated to +-448.  head_dim a multiple of 16.
 */
pkv_status pkv_kv_append_fp8(const void* k_new, const void* v_new, void* k_pool, void* v_pool,
                             const int64_t* slot_mapping, int num_tokens, int num_blocks, int num_kv_heads,
                             int head_dim, int block_size, pkv_dtype src_dtype, float k_scale, float v_scale,
                             void* stream);

/*
 * pkv_paged_attention_decode_fp8 -- pkv_paged_attention_decode over FP8
 * pools: q and out of type dtype (bf16 or f16), K/V values = code x k_scale /
 * x v_scale.  Same workspace as pkv_attention_workspace_bytes.  Runs on
 * tensor cores in FP16 with fp32 accumulation (every code converts exactly;
 * q and the softmax weights are rounded to FP16 once): query groups of 2..16
 * heads share each K/V tile, other group sizes go one query head per warp.
 */
pkv_status pkv_paged_attention_decode_fp8(void* out, const void* q, const void* k_pool, const void* v_pool,
                                          const int32_t* block_tables, int max_blocks_per_seq,
                                          const int32_t* context_lens, int num_seqs, int num_q_heads,
                                          int num_kv_heads, int head_dim, int block_size, int num_blocks,
                                          float scale, float k_scale, float v_scale, int partition_size,
                                          void* workspace, size_t workspace_bytes, pkv_dtype dtype, void* stream);

/*
 * pkv_paged_attention_decode_static -- the same decode attention, for callers
 * that cannot allocate device memory.  The pages have no counterpart to this
 * call; it exists for integration only.
 *
 * Some callers cannot call cudaMalloc or hand in a workspace: a host process
 * whose memory allocator owns all device memory and forbids side
 * allocations, a plug-in limited to the buffers it is given, or a step loop
 * that must not hit a synchronising allocation.  This call takes its split-K
 * scratch from a buffer built into the library instead: 64 MiB of device
 * memory, one per GPU that loads the library, held until the process exits.
 * Arguments and results are those of pkv_paged_attention_decode without the
 * workspace pair; the caller still passes every input and output.
 *   - Size limit: a call whose split-K partials would need more than 64 MiB
 *     (num_seqs * num_q_heads * ceil(max_blocks_per_seq*block_size /
 *     partition) * (head_dim + 2) * 4 bytes) is rejected with
 *     PKV_ERR_INVALID and a message; nothing is launched.
 *   - Set-up: every call that splits its contexts looks up the buffer's
 *     device address on the device current at the call (a CUDA runtime
 *     query that allocates nothing), so a new context on that device is
 *     always served at the right address.  The first such call on a device
 *     may also load the library's device code: make it before any stream
 *     capture.  Calls run on the device that is current when they are made.
 *   - The size limit is checked after every other argument, so an invalid
 *     argument is reported as itself, not as a lack of scratch.
 *   - Sharing: every call on a device uses the same buffer, and it keeps
 *     whatever the last call left in it.  Nothing in it needs to start at
 *     zero.  Calls that overlap on the GPU (different streams, no ordering
 *     between them) race on the buffer and their results are undefined;
 *     order them on one stream or with events.
 *   - The call itself allocates nothing.
 */
pkv_status pkv_paged_attention_decode_static(void* out, const void* q, const void* k_pool, const void* v_pool,
                                             const int32_t* block_tables, int max_blocks_per_seq,
                                             const int32_t* context_lens, int num_seqs, int num_q_heads,
                                             int num_kv_heads, int head_dim, int block_size, int num_blocks,
                                             float scale, int partition_size, pkv_dtype dtype, void* stream);

/*
 * pkv_block_copy -- copy-on-write support: copy whole blocks (every kv head,
 * every offset, K and V) from src to dst ([E] 6.2: only the block being
 * written is copied; the original keeps serving its other users; [B] 2.2).
 *   pairs  int32 [num_pairs][2] = (src, dst) in device memory.  Destinations
 *          must be distinct and none may also be a source.
 * Bit-exact.
 */
pkv_status pkv_block_copy(void* k_pool, void* v_pool, const int32_t* pairs, int num_pairs,
                          int num_blocks, int num_kv_heads, int head_dim, int block_size,
                          pkv_dtype dtype, void* stream);

/*
 * Wait for `stream`, then return the device error word (PKV_DEVERR_* bits)
 * in *code and clear it.  Returns PKV_ERR_DEVICE_CHECK when a bit was set.
 */
pkv_status pkv_device_error(void* stream, uint32_t* code);

/* Number of kernels this library has launched in this process. */
uint64_t pkv_launch_count(void);

/*
 * pkv_step_from_host -- a whole step of the path in one call, for a serving
 * loop that holds each step's inputs and wants its output in host memory.
 * One decode step, as the pages describe it: the step's new K/V are written
 * into the slots the allocator gave them ([E] 2.2, [T] 2.2.3), after the
 * copy-on-write copies of shared blocks being written ([E] 6.2, [B] 2.2), and
 * every query attends to its cache through its block table ([E] 4.2).  On
 * `stream`, in this order:
 *   1. the n_in copies in[i] (typically host -> device: q, the new K/V and the
 *      plan arrays the allocator produced),
 *   2. pkv_block_copy of num_pairs pairs (skipped when num_pairs = 0),
 *   3. pkv_kv_append (PKV_STEP_DECODE_FP8: pkv_kv_append_fp8) of num_tokens
 *      new tokens (skipped when num_tokens = 0),
 *   4. the attention call of `kind` (skipped when num_seqs = 0),
 *   5. the n_out copies out[i] (typically device -> host: the output).
 * Each copy is one cudaMemcpyAsync (cudaMemcpyDefault: the direction follows
 * from the pointers); from pinned host memory it does not wait for the
 * stream.  The device pointers in the struct (pools, pairs, k_new, v_new,
 * slot_mapping, out, q, tables, lengths, groups, query_start, workspace) are
 * the arguments of the separate calls above, with their meaning, layout and
 * checks, and may be the destinations of the copies of step 1.  Sizes are
 * trusted as everywhere else.  Ownership: every buffer is the caller's.
 * Errors: each call checks its own arguments before it launches; the first
 * non-OK status is returned and nothing after it is issued, but what was
 * issued before it (copies, calls) stays issued, so a refused step leaves the
 * pools in an intermediate state -- check a step's arguments once, then reuse
 * them.  struct_size must be sizeof(pkv_step) (PKV_ERR_INVALID otherwise),
 * so a caller built against another version of this header is refused.
 *
 * Overlapped input copies (copy_stream, inputs_free, inputs_ready: all three
 * set, or all three null -- PKV_ERR_INVALID otherwise).  Then step 1's copies
 * go on copy_stream instead of `stream`: copy_stream first waits for
 * inputs_free, the copies follow, inputs_ready is recorded on copy_stream and
 * `stream` waits for it before step 2; inputs_free is recorded on `stream`
 * right after step 4 (after the last of steps 2-4 issued), the point after
 * which no call of this step reads the copies' destinations.  So a step's
 * input copies can run while earlier work on `stream` (a previous step's
 * kernels) still runs, as long as they write other buffers: a caller that
 * alternates sets of destination buffers gives each set its own
 * inputs_free event (so a copy into a set waits only for the last step that
 * read that set) and may share one inputs_ready.  The events are the
 * caller's cudaEvent_t (made with cudaEventDisableTiming or not), the stream
 * its cudaStream_t.
 *
 * Overlapped output copies (out_stream, outputs_done: both set, or both
 * null; they need the input-copy fields set too -- PKV_ERR_INVALID
 * otherwise).  Then step 5's copies go on out_stream instead of `stream`:
 * out_stream waits for inputs_free (recorded after step 4), the copies
 * follow, and outputs_done is recorded on out_stream; before step 4 `stream`
 * waits for outputs_done as last recorded (the previous step whose output
 * copies read the same attention output buffer).  So the next step's kernels
 * on `stream` need not wait for this step's output to cross to the host: a
 * caller that alternates output buffers gives each its own outputs_done.
 * With them the output is in its destination once outputs_done has been
 * reached -- not when `stream` reaches the end of the call -- and
 * out_stream should be another stream than copy_stream (output copies
 * queued there would hold back the next step's input copies).  Without
 * them the output copies stay on `stream`.
 */
typedef struct {
    void* dst;
    const void* src;
    size_t bytes;
} pkv_copy;

typedef enum {
    PKV_STEP_DECODE = 0,         /* pkv_paged_attention_decode */
    PKV_STEP_DECODE_SHARED = 1,  /* pkv_paged_attention_decode_shared */
    PKV_STEP_DECODE_FP8 = 2,     /* pkv_kv_append_fp8 + pkv_paged_attention_decode_fp8 */
    PKV_STEP_CHUNK = 3           /* pkv_paged_attention_chunk (rows = num_tokens) */
} pkv_step_kind;

typedef struct {
    size_t struct_size;          /* sizeof(pkv_step) */
    int kind;                    /* pkv_step_kind */
    const pkv_copy* in;          /* [n_in], made first */
    int n_in;
    const pkv_copy* out;         /* [n_out], made last */
    int n_out;
    /* pools: [num_blocks][num_kv_heads][block_size][head_dim] */
    void* k_pool;
    void* v_pool;
    int num_blocks, num_kv_heads, head_dim, block_size;
    int dtype;                   /* pkv_dtype of q, out and the new K/V (the pools' type unless FP8) */
    float k_scale, v_scale;      /* FP8 pools only */
    /* copy-on-write pairs, int32 [num_pairs][2] */
    const int32_t* pairs;
    int num_pairs;
    /* new tokens: [num_tokens][num_kv_heads][head_dim], int64 slots */
    const void* k_new;
    const void* v_new;
    const int64_t* slot_mapping;
    int num_tokens;
    /* attention */
    void* attn_out;
    const void* q;
    const int32_t* block_tables;
    int max_blocks_per_seq;
    const int32_t* context_lens;
    int num_seqs, num_q_heads;
    float scale;
    int partition_size;
    void* workspace;
    size_t workspace_bytes;
    /* PKV_STEP_DECODE_SHARED */
    const int32_t* group_first;
    const int32_t* group_shared;
    int num_groups, max_group_size, max_shared_len;
    /* PKV_STEP_CHUNK */
    const int32_t* query_start;
    int max_query_len;
    /* overlapped input copies (see above): cudaStream_t, cudaEvent_t, cudaEvent_t, or all null */
    void* copy_stream;
    void* inputs_free;
    void* inputs_ready;
    /* overlapped output copies (see above): cudaStream_t, cudaEvent_t, or both null */
    void* out_stream;
    void* outputs_done;
} pkv_step;

pkv_status pkv_step_from_host(const pkv_step* step, void* stream);

/* --------------------------------------------------------- host allocator */

/*
 * Host block allocator: free pool, per-block reference counts, per-sequence
 * block tables, shared prefixes, forks and the copy-on-write trigger
 * ([E] 4.1-4.3, 6.1-6.2; [B] 2.1-2.2, 3.1; [T] 2.2.2-2.2.3, 2.2.13).
 * The handle is owned by the library; one handle must not be used from two
 * threads at once.  Every call is all-or-nothing: on any error the state is
 * unchanged.  Policy: the free pool is a FIFO queue; a new block is taken
 * from its front only when a sequence's last block is full; freed blocks go
 * to its back in block-table order.
 */
typedef struct pkv_alloc pkv_alloc;

/* free_order: a permutation of 0..num_blocks-1 giving the initial queue, or NULL for 0,1,2,... */
pkv_alloc* pkv_alloc_create(int num_blocks, int block_size, const int32_t* free_order);
void pkv_alloc_destroy(pkv_alloc* a);

/* Register an empty sequence. */
pkv_status pkv_seq_add(pkv_alloc* a, int64_t seq_id);

/*
 * Point an empty, registered sequence at existing blocks holding its first
 * `num_tokens` tokens (a shared system prompt: [E] 6.1, [T] 2.2.3).
 * nblocks must equal ceil(num_tokens/block_size); blocks must be distinct and
 * currently in use.  Each block's reference count goes up by one.
 */
pkv_status pkv_seq_share_prefix(pkv_alloc* a, int64_t seq_id, const int32_t* blocks, int nblocks,
                                int num_tokens);

/* New sequence `child` sharing every block of `parent` ([B] 2.2). */
pkv_status pkv_seq_fork(pkv_alloc* a, int64_t parent, int64_t child);

/*
 * Reserve slots for `ntok` new tokens of a sequence.
 *   slots_out  int64 [ntok]: the slot of each new token, in order.
 *   cow_out    int32 [cow_cap][2]: (src, dst) block pairs the caller must copy
 *              (pkv_block_copy) before writing the new tokens; at most one
 *              per call, so cow_cap >= 1 suffices.  *n_cow = pairs written.
 * A fresh block is taken when the last block is full; if the token lands in a
 * block whose reference count is above one (or, with prefix caching, a cached
 * block), that block alone is copied to a fresh block and replaced in this
 * sequence's table ([E] 6.2).  PKV_ERR_NO_FREE_BLOCK if the pool runs out
 * (counted in alloc_failures); the call then changes nothing else.
 */
pkv_status pkv_seq_append_slots(pkv_alloc* a, int64_t seq_id, int ntok, int64_t* slots_out,
                                int32_t* cow_out, int cow_cap, int* n_cow);

/*
 * One decode step's host work for many sequences in one call: reserve one
 * slot for each of seq_ids[0..n-1], in that order, exactly as n calls of
 * pkv_seq_append_slots(a, seq_ids[i], 1, ...) would.
 *   slots_out  int64 [n]
 *   cow_out    int32 [cow_cap][2]; *n_cow = pairs written (at most n).
 * All-or-nothing: if any sequence fails (unknown id, pool exhausted, cow_cap
 * too small), nothing changes and *n_cow = 0 (an exhausted pool still counts
 * one allocation failure in pkv_alloc_stats).  Blocks are counted in call
 * order, so a step that the n single calls complete is never refused.
 */
pkv_status pkv_seq_append_slots_batch(pkv_alloc* a, const int64_t* seq_ids, int n, int64_t* slots_out,
                                      int32_t* cow_out, int cow_cap, int* n_cow);

/*
 * Block tables and lengths of many sequences: row i of out (int32 [n][max_blocks])
 * gets seq_ids[i]'s table padded with -1, lens_out[i] its length in tokens.
 * PKV_ERR_INVALID (nothing written) if a sequence is unknown or longer than
 * max_blocks blocks.
 */
pkv_status pkv_seq_block_tables_batch(const pkv_alloc* a, const int64_t* seq_ids, int n, int32_t* out,
                                      int max_blocks, int32_t* lens_out);

/*
 * Lengths in tokens of many sequences, without their tables: lens_out[i]
 * (int64 [n]) = seq_ids[i]'s length.  PKV_ERR_INVALID (nothing written) if a
 * sequence is unknown.  A host-side check before a step (will every sequence
 * still fit its table?) needs only these.
 */
pkv_status pkv_seq_lens_batch(const pkv_alloc* a, const int64_t* seq_ids, int n, int64_t* lens_out);

/*
 * Automatic prefix caching ([E] 7.4: a prompt prefix computed once is reused
 * by later requests, which skip that part of the prefill; [T] 2.2.3 shared
 * blocks, 2.2.8 only byte-identical prefixes may share, 2.2.13 hit rate).
 * Off by default; switch it on before any sequence is registered.  With it
 * on: every full block filled through pkv_seq_append_tokens or
 * pkv_seq_add_with_prompt is keyed by its block_size token ids plus the key
 * of the block before it (exact equality, no hashing of content), so a key
 * match means an identical whole prefix; a block whose count drops to zero
 * stays cached (evictable, least recently released first) and counts as
 * free; a fresh block comes from the free queue first, then by evicting the
 * oldest evictable block.  Appending without token ids (pkv_seq_append_slots,
 * _batch) or sharing by block list stops a sequence from registering blocks.
 * A cached block is never written in place: a sequence that holds one with
 * fewer of its tokens (a prefix shared part-way into it) gets a copy-on-write
 * pair for it, as when another sequence holds it.
 */
pkv_status pkv_alloc_set_prefix_caching(pkv_alloc* a, int enable);

/*
 * Register a new sequence with its prompt tokens[0..ntok-1]: the longest run
 * of cached full blocks matching the prompt's leading blocks is reused (their
 * K/V need not be computed), the rest get fresh slots.  *n_cached = tokens
 * reused (a multiple of block_size); slots_out[0 .. ntok-*n_cached-1] = slots
 * of the remaining tokens, for pkv_kv_append.  All-or-nothing.
 */
pkv_status pkv_seq_add_with_prompt(pkv_alloc* a, int64_t seq_id, const int32_t* tokens, int ntok,
                                   int64_t* slots_out, int* n_cached);

/* pkv_seq_append_slots with the new tokens' ids, so that blocks they fill get cached. */
pkv_status pkv_seq_append_tokens(pkv_alloc* a, int64_t seq_id, const int32_t* tokens, int ntok,
                                 int64_t* slots_out, int32_t* cow_out, int cow_cap, int* n_cow);

/* Prefix-cache counters: full prompt blocks looked up, found, cached now,
 * evictable now, evicted so far.  Any pointer may be NULL. */
pkv_status pkv_prefix_cache_stats(const pkv_alloc* a, int64_t* lookups, int64_t* hits, int* cached_blocks,
                                  int* evictable_blocks, int64_t* evictions);

/* Drop a sequence; blocks whose count reaches zero return to the free pool ([T] 2.2.2). */
pkv_status pkv_seq_free(pkv_alloc* a, int64_t seq_id);

/*
 * Copy a sequence's block table into out[cap]; *n = its number of blocks
 * (PKV_ERR_INVALID if cap < *n, with *n still set), *len_tokens = its length.
 */
pkv_status pkv_seq_block_table(const pkv_alloc* a, int64_t seq_id, int32_t* out, int cap, int* n,
                               int64_t* len_tokens);

/* Pool occupancy and counters for monitoring ([T] 2.2.13). Any pointer may be NULL. */
pkv_status pkv_alloc_stats(const pkv_alloc* a, int* free_blocks, int* used_blocks,
                           int64_t* alloc_failures, int64_t* cow_copies);

/* Reference count of a block, or -1 if the id is out of range. */
int pkv_block_refcount(const pkv_alloc* a, int block);

/* ------------------------------------------------------------------ misc */
const char* pkv_status_str(pkv_status s);
/* Message describing the last failed call on this thread ("" if none). */
const char* pkv_last_error(void);

#ifdef __cplusplus
}
#endif
#endif /* PAGEDKV_H */
