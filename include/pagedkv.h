/*
 * pagedkv.h - C ABI of libpagedkv: PagedAttention's data-parallel decode path
 * on NVIDIA B200 (sm_100a), plus the host block manager that feeds it.
 *
 * Sources (web pages on PagedAttention, cited by page title and section):
 *   [Q] "What is PagedAttention?" (qubittool.com glossary), How It Works:
 *       Map Logical to Physical Blocks; Share Without Mutating State.
 *   [K] "PagedAttention" (kongchang.com knowledge page), Core Facts.
 *   [G] "PagedAttention: Optimizing KV Cache in vLLM" (grasp.study lesson),
 *       section 2 (The Solution), section 3 (Making it Work: The PagedAttention
 *       Kernel), section 4 (Zero-Cost Sharing with Copy-on-Write).
 *
 * Conventions for every call below
 * --------------------------------
 * - All tensors are caller-owned. Device pointers must point to memory on the
 *   current CUDA device; the library never frees or keeps them after return.
 *   No kernel entry point allocates device memory.
 * - Every kernel entry point enqueues work on `stream` (a cudaStream_t passed
 *   as void*; NULL is the legacy default stream) and returns without
 *   synchronising. A PA_OK return means the launch was accepted.
 * - Layouts (row-major, contiguous, no padding):
 *     k_pool, v_pool : [num_blocks][num_kv_heads][block_size][head_dim]
 *                      One (physical block, KV head) tile is contiguous.
 *     q, out         : [num_seqs][num_q_heads][head_dim]
 *     block_tables   : int32 [num_seqs][max_blocks_per_seq]; entry [s][i] is the
 *                      physical block of logical block i of sequence s [Q].
 *                      Entries at or past ceil(ctx_s / block_size) are never read.
 *     context_lens   : int32 [num_seqs], tokens held by each sequence.
 *     slot_mapping   : int64 [num_tokens], slot = block * block_size + offset;
 *                      a negative slot is padding and writes nothing.
 * - Query head h reads KV head h / (num_q_heads / num_kv_heads): consecutive
 *   query heads share one KV head (grouped-query attention, [K]).
 * - dtype is PA_F32 (all of q, pools, out fp32) or PA_BF16 (all bf16);
 *   arithmetic is fp32 in both cases. out has q's dtype.
 * - Supported shapes: head_dim in {64, 128, 256} (256 for bf16 only),
 *   block_size in {16, 32}; bf16 takes any group size 1..16, fp32 takes group
 *   sizes 1, 2, 4, 8. bf16 products run on tensor cores (P rounded to bf16
 *   before P*V, fp32 accumulation); fp32 runs on CUDA cores.
 *   num_blocks * num_kv_heads * block_size < 2^31.
 *   Pointers to pools, q, out, k_new and v_new must be 16-byte aligned.
 * - Errors: invalid arguments are rejected before anything is enqueued
 *   (PA_ERR_INVALID_ARG / PA_ERR_UNSUPPORTED, nothing changes). Kernels never
 *   trap: an index found out of range on the device (a block id outside
 *   [0, num_blocks), a context length outside [0, max_blocks_per_seq *
 *   block_size], a slot past the pool) sets a PA_DEVERR_* bit in *dev_err (when
 *   dev_err is non-NULL, atomically OR-ed, never cleared by the library) and
 *   the offending access is skipped. The text of the last host-side error of
 *   the calling thread is returned by pa_last_error_string().
 */
#ifndef PAGEDKV_H_
#define PAGEDKV_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  PA_OK = 0,
  PA_ERR_INVALID_ARG = 1,     /* bad pointer, size, shape or alignment */
  PA_ERR_NO_FREE_BLOCKS = 2,  /* block manager out of blocks; state unchanged */
  PA_ERR_CUDA = 3,            /* a CUDA runtime/driver call failed */
  PA_ERR_UNSUPPORTED = 4      /* valid request outside the compiled shapes */
} pa_status_t;

typedef enum { PA_F32 = 0, PA_BF16 = 1 } pa_dtype_t;

/* Bits OR-ed into the optional device error word. */
#define PA_DEVERR_BLOCK_ID 0x1u     /* block table entry outside [0, num_blocks) */
#define PA_DEVERR_CONTEXT_LEN 0x2u  /* context length < 0 or > max_blocks_per_seq*block_size */
#define PA_DEVERR_SLOT 0x4u         /* slot >= num_blocks * block_size */
#define PA_DEVERR_COPY_PAIR 0x8u    /* copy pair index outside [0, num_blocks) */
#define PA_DEVERR_TIMEOUT 0x10u     /* a pipeline wait hit its time limit; output invalid */

/* Library version string, e.g. "pagedkv 0.1 sm_100a". */
const char* pa_version(void);
/* Text of the last error reported to the calling thread ("" if none). */
const char* pa_last_error_string(void);
/* Static name of a status code. */
const char* pa_status_string(pa_status_t status);

/* ---------------------------------------------------------------------------
 * pa_decode - single-query decode attention over the paged KV cache.
 *
 * For every sequence s and query head h:
 *     out[s][h] = softmax(scale * K_s q[s][h]) V_s
 * where K_s, V_s are the first context_lens[s] tokens of KV head
 * h / (num_q_heads / num_kv_heads), gathered in logical order through
 * block_tables[s]. The kernel walks the blocks in logical order with a
 * running-max softmax, so the result equals attention over a contiguous copy
 * of the sequence ([G] section 3; the table indirection is [Q], Map Logical to
 * Physical Blocks). A sequence with context length 0 gets zeros.
 *
 * One CTA per (sequence, KV head) handles the whole context; for long or
 * ragged contexts prefer pa_decode_split.
 * ------------------------------------------------------------------------- */
pa_status_t pa_decode(const void* q, const void* k_pool, const void* v_pool,
                      const int32_t* block_tables, const int32_t* context_lens,
                      int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                      int block_size, int num_blocks, int max_blocks_per_seq,
                      float scale, pa_dtype_t dtype, void* out, uint32_t* dev_err,
                      void* stream);

/* ---------------------------------------------------------------------------
 * pa_decode_split - the same result as pa_decode, computed by cutting the
 * contexts into pieces. Each (sequence, KV head, piece) produces a running
 * max, a running sum and an unnormalised accumulator; a log-sum-exp merge
 * combines the pieces, and a sequence held in one piece is written directly.
 * The split is a scheduling device for long and ragged contexts; it does not
 * appear on the pages, which only require that the blockwise walk reproduce
 * the contiguous result ([G] section 3). Two cuts, chosen by the table size:
 *  - tables of fewer than 32768 tokens (max_blocks_per_seq * block_size):
 *    partitions of partition_tokens tokens (a multiple of block_size),
 *    handed to persistent CTAs as work tickets;
 *  - longer tables: every warp of a persistent grid takes an equal run of
 *    16-token units of one KV head's work, sequence after sequence, so the
 *    piece boundaries follow the whole batch; partition_tokens then only
 *    bounds the pieces: no (sequence, KV head) is cut into more than
 *    ceil(max_blocks_per_seq / (partition_tokens / block_size)) + 1.
 *   (PAGEDKV_SPLIT_KERNEL=ticket|stream forces one cut.) Both give the
 *   contiguous result to rounding; with the second, the rounding of one
 *   sequence can depend on the rest of the batch. Same inputs give the same
 *   bits.
 *
 * workspace: caller-owned device memory of at least
 *   pa_decode_split_workspace_size(...) bytes, 256-byte aligned. It starts
 *   with a 256-byte control header (work-ticket counters) that must be zero
 *   before the first call; pa_decode_split_workspace_init zeroes the whole
 *   workspace. Every completed call leaves the header zero again, so one
 *   workspace serves any number of calls issued in stream order. Calls that
 *   may overlap on the GPU need separate workspaces. After a call that
 *   reported PA_DEVERR_TIMEOUT, initialise the workspace again.
 * Two kernels run: the decode kernel, then the merge kernel, launched as a
 *   programmatic dependent so that it waits on the device rather than in the
 *   launch queue (rows held in one piece return at once).
 * num_seqs must be <= 4096 (PA_ERR_UNSUPPORTED above that).
 * ------------------------------------------------------------------------- */
size_t pa_decode_split_workspace_size(int num_seqs, int num_q_heads, int head_dim,
                                      int block_size, int max_blocks_per_seq,
                                      int partition_tokens);

pa_status_t pa_decode_split_workspace_init(void* workspace, size_t workspace_bytes,
                                           void* stream);

pa_status_t pa_decode_split(const void* q, const void* k_pool, const void* v_pool,
                            const int32_t* block_tables, const int32_t* context_lens,
                            int num_seqs, int num_q_heads, int num_kv_heads,
                            int head_dim, int block_size, int num_blocks,
                            int max_blocks_per_seq, float scale, pa_dtype_t dtype,
                            int partition_tokens, void* workspace,
                            size_t workspace_bytes, void* out, uint32_t* dev_err,
                            void* stream);

/* ---------------------------------------------------------------------------
 * pa_decode_split_static - pa_decode_split for callers that cannot allocate
 * device memory. (Not from the pages: the paper has no counterpart; this is
 * an interface convenience of this library.)
 *
 * Some callers have no way to call cudaMalloc: their device memory is owned
 * by another allocator (a framework's caching allocator or a fixed arena
 * sized up front), or they run where an allocation that may synchronise the
 * device or fail halfway through a decode loop is not acceptable. This entry
 * point takes the same inputs and output as pa_decode_split, minus the
 * workspace: its scratch (ticket counters and per-partition partials) lives
 * in a fixed array of PA_STATIC_SCRATCH_BYTES inside the library's device
 * image, which every GPU that loads the library holds until the process
 * exits. It allocates no device memory and calls no allocating routine.
 *
 * - Sizes whose scratch would exceed PA_STATIC_SCRATCH_BYTES (see
 *   pa_decode_split_workspace_size) are rejected with PA_ERR_INVALID_ARG and
 *   a message naming both sizes, before anything is enqueued. Every other
 *   refusal (bad arguments, more than 4096 sequences, PAGEDKV_VALIDATE
 *   findings) also happens before the array is touched.
 * - The first call in each CUDA context (with that context, and so its
 *   device, current) looks up the array's device address
 *   (cudaGetSymbolAddress) and caches it, keyed by the context: an address
 *   is only valid in the context it was taken in. Make that first call
 *   before any stream capture.
 * - All calls on a device share the one array, and it keeps the previous
 *   call's contents. Each accepted call clears the part that must start at
 *   zero (on `stream`, right before its kernels). Calls that may overlap on
 *   the GPU (other streams, other host threads) race on the array and must
 *   be serialised by the caller; calls issued in order on one stream are
 *   safe.
 * ------------------------------------------------------------------------- */
#define PA_STATIC_SCRATCH_BYTES (16u * 1024u * 1024u)

pa_status_t pa_decode_split_static(const void* q, const void* k_pool, const void* v_pool,
                                   const int32_t* block_tables, const int32_t* context_lens,
                                   int num_seqs, int num_q_heads, int num_kv_heads,
                                   int head_dim, int block_size, int num_blocks,
                                   int max_blocks_per_seq, float scale, pa_dtype_t dtype,
                                   int partition_tokens, void* out, uint32_t* dev_err,
                                   void* stream);

/* Test aid for the contract above: sets every byte of the static scratch's
 * control header (its first 256 bytes, the ticket counters) to `byte` on
 * `stream`, in the current context, as a call that ended early (a device
 * timeout) could leave it. The next pa_decode_split_static call must still
 * be correct, since each call clears the header after its host checks.
 * Enqueues one memset; allocates nothing. */
pa_status_t pa_decode_split_static_fill_header(uint8_t byte, void* stream);

/* ---------------------------------------------------------------------------
 * pa_decode_shared_prefix - the same result as pa_decode, reading each
 * shared prefix once. Sequences that share their first blocks (prefix
 * sharing and parallel sampling, [G] section 4; [Q] Share Without Mutating
 * State) are given as groups: group g lists positions group_members
 * [group_offsets[g] .. group_offsets[g+1]) of the batch, which all hold the
 * same physical blocks in table entries 0 .. group_blocks[g]-1, every one of
 * them full (pa_bm_prefix_groups produces exactly this). A prefix kernel
 * streams each group's shared blocks once per KV head for all of the group's
 * query rows (members x heads per KV head, on tensor cores); the split kernel
 * then covers each sequence's remaining blocks; the log-sum-exp merge joins
 * the two ([G] section 3: any blockwise order gives the contiguous result).
 * Sequences in no group are decoded as by pa_decode_split.
 *
 * Group arrays are HOST memory, read during the call; the library copies what
 * the kernels need into the workspace. bf16 only. workspace: at least
 * pa_decode_shared_prefix_workspace_size(...) bytes, 256-byte aligned,
 * initialised once with pa_decode_split_workspace_init (the same contract as
 * pa_decode_split).
 *
 * Host plans (this call and pa_prefill): the plan built from the host
 * arrays reaches the device on `stream` without the call waiting for the
 * stream. A plan of up to 30 KB (a few hundred work items) travels as the
 * parameters of a small kernel, so the call may be captured into a CUDA
 * graph: a replay uploads the plan captured with it. A larger plan is copied
 * into a page-locked staging slot owned by the library and uploaded from
 * there; slots are reused once their upload has completed, so such a call
 * is refused with PA_ERR_UNSUPPORTED while `stream` is being captured (a
 * replay would read a slot that has since been reused), before anything is
 * enqueued.
 * ------------------------------------------------------------------------- */
size_t pa_decode_shared_prefix_workspace_size(int num_seqs, int num_q_heads, int num_kv_heads,
                                              int head_dim, int block_size,
                                              int max_blocks_per_seq, int partition_tokens);

pa_status_t pa_decode_shared_prefix(const void* q, const void* k_pool, const void* v_pool,
                                    const int32_t* block_tables, const int32_t* context_lens,
                                    int num_seqs, int num_q_heads, int num_kv_heads,
                                    int head_dim, int block_size, int num_blocks,
                                    int max_blocks_per_seq, float scale, pa_dtype_t dtype,
                                    int partition_tokens, int num_groups,
                                    const int32_t* group_offsets, const int32_t* group_members,
                                    const int32_t* group_blocks, void* workspace,
                                    size_t workspace_bytes, void* out, uint32_t* dev_err,
                                    void* stream);

/* ---------------------------------------------------------------------------
 * pa_decode_split_window - sliding-window decode: as pa_decode_split, but
 * each query attends only to the last `window` tokens of its sequence
 * (tokens max(0, ctx - window) .. ctx - 1; window >= 1). The block walk
 * starts at the window's first block and the tokens before the window in
 * that block are masked, so table entries before it are never read and may
 * be -1 (pa_bm_release_before). Sliding-window attention is named beside
 * paged attention as a KV-cache optimisation ([K] Core Facts). Same
 * workspace and contract as pa_decode_split.
 * ------------------------------------------------------------------------- */
pa_status_t pa_decode_split_window(const void* q, const void* k_pool, const void* v_pool,
                                   const int32_t* block_tables, const int32_t* context_lens,
                                   int num_seqs, int num_q_heads, int num_kv_heads,
                                   int head_dim, int block_size, int num_blocks,
                                   int max_blocks_per_seq, float scale, pa_dtype_t dtype,
                                   int partition_tokens, int window, void* workspace,
                                   size_t workspace_bytes, void* out, uint32_t* dev_err,
                                   void* stream);

/* ---------------------------------------------------------------------------
 * pa_prefill - causal (chunked) prefill attention over the paged cache.
 * Sequence s holds context_lens[s] tokens, the last query_lens[s] of them
 * new (their K and V already written, e.g. by pa_kv_append); its queries are
 * rows query_start .. query_start + query_lens[s] - 1 of q
 * [total_q][num_q_heads][head_dim] (sequences back to back, total_q = sum of
 * query_lens). New token i at position p = ctx - qlen + i attends to tokens
 * 0..p of its sequence through its block table; out has q's layout. Prefill
 * is the step that fills a request's first blocks ([Q] How It Works: prefill
 * allocates enough blocks for the input).
 *
 * context_lens and query_lens are HOST arrays here (the host plans the
 * tiles); block tables are device memory. bf16, head_dim 64 or 128, block
 * size 16 or 32. Each CTA takes two tiles of 128 query rows (query tokens x
 * heads of one KV head; tcgen05 tensor cores, accumulators in tensor
 * memory; PAGEDKV_PREFILL_KERNEL=mma_sync selects 64-row mma.sync tiles)
 * and reads their KV once per partition of partition_tokens tokens; tiles
 * spanning several partitions are joined by the log-sum-exp merge. With
 * more (tile pair, partition) items than resident CTAs the tcgen05 kernel
 * runs persistently: the host hands each item to the CTA with the least
 * estimated work so far, and a CTA loads its next item's Q and K/V while it
 * finishes the current one (PAGEDKV_PREFILL_CTAS=n caps that grid). q and
 * out must be 16-byte aligned; with total_q = 0 they may be NULL and the
 * call enqueues nothing. workspace: at least pa_prefill_workspace_size(...)
 * bytes, 256-byte aligned, initialised once with
 * pa_decode_split_workspace_init.
 * ------------------------------------------------------------------------- */
size_t pa_prefill_workspace_size(int num_seqs, int total_q, int num_q_heads, int num_kv_heads,
                                 int head_dim, int block_size, int max_blocks_per_seq,
                                 int partition_tokens);

pa_status_t pa_prefill(const void* q, const void* k_pool, const void* v_pool,
                       const int32_t* block_tables, const int32_t* context_lens,
                       const int32_t* query_lens, int num_seqs, int total_q, int num_q_heads,
                       int num_kv_heads, int head_dim, int block_size, int num_blocks,
                       int max_blocks_per_seq, float scale, pa_dtype_t dtype,
                       int partition_tokens, void* workspace, size_t workspace_bytes, void* out,
                       uint32_t* dev_err, void* stream);

/* ---------------------------------------------------------------------------
 * pa_prefill_plan - the work plan pa_prefill makes for its tcgen05 kernel,
 * for inspection and tests; host only (no CUDA call, no device needed).
 * Items are (sequence, run of query tokens, KV head, KV partition): one per
 * partition of partition_tokens tokens of each KV head of each run of
 * 2 x (128 / group) query tokens, in sequence order with each sequence's
 * runs last-first. With max_ctas > 0 and more items than max_ctas, the
 * items are scheduled over max_ctas CTAs: each goes, in that order, to the
 * CTA with the least estimated work so far (ties to the lowest CTA), and
 * the items are listed CTA by CTA, each CTA's in that order (the order the
 * kernel runs them). Otherwise item i runs on CTA i.
 *
 * context_lens, query_lens: HOST int32 [num_seqs] (as for pa_prefill).
 * num_items, num_ctas: out, the item count and the grid. items_out: NULL
 * (counts only) or HOST int32 [max_items][6] rows (seq, first query token,
 * query tokens, kv head, partition, cta); max_items below the item count is
 * PA_ERR_INVALID_ARG. block_size 16 or 32, else PA_ERR_UNSUPPORTED.
 * pa_prefill plans the same way, with max_ctas = the kernel's resident CTAs
 * (capped by PAGEDKV_PREFILL_CTAS).
 * ------------------------------------------------------------------------- */
pa_status_t pa_prefill_plan(const int32_t* context_lens, const int32_t* query_lens, int num_seqs,
                            int num_q_heads, int num_kv_heads, int block_size, int partition_tokens,
                            int max_ctas, int32_t* items_out, int max_items, int* num_items,
                            int* num_ctas);

/* ---------------------------------------------------------------------------
 * pa_swap_out / pa_swap_in - the data movement of swapping: whole blocks
 * (K and V, all heads; block_bytes each) between the device pools and two
 * host buffers of num_host_slots blocks each. pairs (device int64
 * [num_pairs][2]): swap-out (device block, host slot), swap-in (host slot,
 * device block). The host buffers must be page-locked and mapped
 * (cudaHostAlloc / cudaHostRegister; the library looks up their device
 * addresses); the copies are kernels that read or write them directly over
 * the host link, 16-byte vectors. Bit-exact. Indices out of range set
 * PA_DEVERR_COPY_PAIR and are skipped.
 * ------------------------------------------------------------------------- */
pa_status_t pa_swap_out(const void* k_pool, const void* v_pool, void* host_k, void* host_v,
                        const int64_t* pairs, int num_pairs, size_t block_bytes, int num_blocks,
                        int num_host_slots, uint32_t* dev_err, void* stream);
pa_status_t pa_swap_in(const void* host_k, const void* host_v, void* k_pool, void* v_pool,
                       const int64_t* pairs, int num_pairs, size_t block_bytes, int num_blocks,
                       int num_host_slots, uint32_t* dev_err, void* stream);

/* ---------------------------------------------------------------------------
 * pa_kv_append - decode-step write of new tokens' keys and values into their
 * slots ([Q], Map Logical to Physical Blocks: decode appends into the partly
 * filled tail block; [G] section 4 step 3: the write proceeds on the private
 * block). k_new, v_new: [num_tokens][num_kv_heads][head_dim] in `dtype`.
 * Token t goes to block slot/block_size, offset slot%block_size, every KV head.
 * Bit-exact copy. Slots must be unique within a call (duplicates race).
 * ------------------------------------------------------------------------- */
pa_status_t pa_kv_append(const void* k_new, const void* v_new,
                         const int64_t* slot_mapping, int num_tokens,
                         int num_kv_heads, int head_dim, int block_size,
                         int num_blocks, pa_dtype_t dtype, void* k_pool,
                         void* v_pool, uint32_t* dev_err, void* stream);

/* ---------------------------------------------------------------------------
 * pa_copy_blocks - the data movement of copy-on-write: for each pair
 * (src, dst) in src_dst_pairs (int64 [num_pairs][2], device memory), copy the
 * whole physical block (block_bytes = num_kv_heads*block_size*head_dim*elt
 * bytes, a multiple of 16) from src to dst in both pools ([G] section 4 step
 * 3; [Q], Share Without Mutating State). Pairs must not chain (no dst is
 * another pair's src) and dst ids must be unique: all pairs are copied at
 * once, in no order, so a list that breaks either rule has an undefined
 * result. Lists from the block manager always keep both (each copy goes to
 * a block it has just taken from the free queue). With PAGEDKV_VALIDATE=1
 * the pairs are read back (synchronously) and such a list, or a pair outside
 * [0, num_blocks), is refused with PA_ERR_INVALID_ARG before any copy.
 * ------------------------------------------------------------------------- */
pa_status_t pa_copy_blocks(void* k_pool, void* v_pool, const int64_t* src_dst_pairs,
                           int num_pairs, size_t block_bytes, int num_blocks,
                           uint32_t* dev_err, void* stream);

/* ===========================================================================
 * Host block manager ([Q] How It Works; [G] sections 2 and 4).
 *
 * An opaque handle owned by the caller (pa_bm_destroy frees it). Not
 * thread-safe: one thread at a time per handle. Sequence ids are any int64.
 * Every call is all-or-nothing: on any error status nothing changes.
 *
 * Policy (the pages leave it open): free blocks form a FIFO queue seeded from
 * initial_free_order (identity when NULL); allocation pops the front; a free
 * call returns the blocks it reclaims to the back in ascending id order.
 * ========================================================================= */
typedef struct pa_bm* pa_bm_t;

typedef struct {
  int64_t num_blocks;
  int64_t free_blocks;
  int64_t used_blocks;      /* blocks with reference count > 0 */
  int64_t shared_blocks;    /* blocks with reference count > 1 */
  int64_t num_seqs;
  int64_t logical_tokens;   /* sum of context lengths */
  int64_t logical_slots;    /* sum of table lengths * block_size */
  int64_t tail_waste_slots; /* logical_slots - logical_tokens */
  int64_t cow_copies;       /* copy-on-write copies made so far */
} pa_bm_stats_t;

/* Create a manager for a pool of num_blocks blocks of block_size tokens; a
 * sequence may hold at most max_blocks_per_seq blocks. initial_free_order, if
 * given, is a permutation of 0..num_blocks-1 (host memory, copied). */
pa_status_t pa_bm_create(int num_blocks, int block_size, int max_blocks_per_seq,
                         const int32_t* initial_free_order, pa_bm_t* out);
pa_status_t pa_bm_destroy(pa_bm_t bm);

/* Prefill: a new sequence with num_tokens tokens takes ceil(num_tokens /
 * block_size) blocks ([Q]). PA_ERR_NO_FREE_BLOCKS if the pool cannot supply
 * them; PA_ERR_INVALID_ARG for an existing id or more than max_blocks_per_seq. */
pa_status_t pa_bm_allocate(pa_bm_t bm, int64_t seq_id, int64_t num_tokens);

/* Sharing: child gets the parent's table and context length; every block's
 * reference count goes up by one; no data moves ([G] section 4 step 1). */
pa_status_t pa_bm_fork(pa_bm_t bm, int64_t parent_id, int64_t child_id);

/* Decode step for one sequence: reserve the slot of its next token. A full
 * (or absent) tail takes a new block; a partly filled tail held by more than
 * one sequence is copied first: a new block is taken, *cow_src/*cow_dst name
 * the copy the caller must perform (pa_copy_blocks) before writing, only this
 * sequence's table changes and the shared block's count drops by one ([G]
 * section 4 steps 2-3). Otherwise *cow_src = *cow_dst = -1. */
pa_status_t pa_bm_append_slot(pa_bm_t bm, int64_t seq_id, int64_t* slot,
                              int64_t* cow_src, int64_t* cow_dst);

/* The same for n distinct sequences in the given order, all or nothing.
 * slots: int64 [n]. cow_pairs: int64 [n][2] receives the copies made, packed
 * at the front; *num_cow (may be NULL) receives their count. */
pa_status_t pa_bm_append_slots(pa_bm_t bm, const int64_t* seq_ids, int n,
                               int64_t* slots, int64_t* cow_pairs, int* num_cow);

/* *ok = 1 if pa_bm_append_slots(seq_ids, n) would succeed now, else 0. */
pa_status_t pa_bm_can_append(pa_bm_t bm, const int64_t* seq_ids, int n, int* ok);

/* Finish a sequence: counts drop by one; blocks reaching zero are reclaimed. */
pa_status_t pa_bm_free(pa_bm_t bm, int64_t seq_id);

/* Sliding window: drop the sequence's references to blocks whose tokens all
 * lie before first_token (blocks 0 .. first_token/block_size - 1). Their table
 * entries become -1, so logical positions stay where they were; blocks whose
 * count reaches zero are reclaimed (back of the free queue, ascending).
 * *num_reclaimed (may be NULL) gets how many. Decode with a window of
 * ctx - first_token tokens or fewer never reads the released entries. */
pa_status_t pa_bm_release_before(pa_bm_t bm, int64_t seq_id, int64_t first_token,
                                 int* num_reclaimed);

/* Preemption by swap ([Q] How It Works: an allocation failure is met by
 * admission control, preemption, swap or rejection). pa_bm_swap_out gives up
 * the sequence's blocks (counts drop by one, blocks reaching zero are
 * reclaimed) but keeps its context length; blocks[0..*n) receives its table
 * at that moment (-1 for released entries). Copy those blocks to host memory
 * (pa_swap_out) on the stream before any later work can reuse them. A
 * swapped-out sequence cannot append, fork or release until pa_bm_swap_in,
 * which takes one new private block per resident entry (all or nothing,
 * PA_ERR_NO_FREE_BLOCKS otherwise) and writes the new table to blocks[0..*n);
 * copy the host copies into those blocks (pa_swap_in) before decoding it. */
pa_status_t pa_bm_swap_out(pa_bm_t bm, int64_t seq_id, int32_t* blocks, int capacity, int* n);
pa_status_t pa_bm_swap_in(pa_bm_t bm, int64_t seq_id, int32_t* blocks, int capacity, int* n);

/* Copy one sequence's block table into row[0..row_capacity); *n_blocks gets
 * its length (PA_ERR_INVALID_ARG if row_capacity is too small). */
pa_status_t pa_bm_block_table(pa_bm_t bm, int64_t seq_id, int32_t* row,
                              int row_capacity, int* n_blocks);
pa_status_t pa_bm_context_len(pa_bm_t bm, int64_t seq_id, int64_t* context_len);

/* Export a batch: tables int32 [n][max_blocks_per_seq] (unused entries set to
 * pad_value) and context_lens int32 [n], both host memory, ready to upload
 * for pa_decode. */
pa_status_t pa_bm_export(pa_bm_t bm, const int64_t* seq_ids, int n, int32_t* tables,
                         int32_t* context_lens, int32_t pad_value);

/* Shared-prefix groups of a batch, for pa_decode_shared_prefix. Sequences
 * whose block tables start with the same physical blocks (created by fork,
 * [G] section 4 step 1) form a group; its shared length is the longest
 * common table prefix, counted in blocks that are full for every member
 * (a partly filled shared tail is left to each sequence). Only groups of at
 * least two sequences sharing at least min_shared_blocks blocks are kept.
 * Outputs (host memory, capacities n+1 / n / n): group_offsets[g] ..
 * group_offsets[g+1] index group_members, which lists positions in seq_ids
 * (in seq_ids order); group_blocks[g] is the shared block count. */
pa_status_t pa_bm_prefix_groups(pa_bm_t bm, const int64_t* seq_ids, int n, int min_shared_blocks,
                                int32_t* group_offsets, int32_t* group_members,
                                int32_t* group_blocks, int* num_groups);

pa_status_t pa_bm_refcount(pa_bm_t bm, int block_id, int* refcount);
/* Free queue front to back into out[0..capacity); *n gets its length. */
pa_status_t pa_bm_free_queue(pa_bm_t bm, int32_t* out, int capacity, int* n);
pa_status_t pa_bm_stats(pa_bm_t bm, pa_bm_stats_t* stats);

/* ===========================================================================
 * pa_decode_step - one whole decode step from host buffers: the block
 * manager reserves one slot per sequence (copy-on-write where a tail is
 * shared), the step's inputs are uploaded, the copies, the KV append and the
 * split decode run, and the output is downloaded. This is call stack A of the
 * pages' flow in one call: decode appends into the tail block ([Q] How It
 * Works), shared tails are copied before the write ([G] section 4), attention
 * walks the block tables ([G] section 3).
 *
 * All buffers in pa_step_buffers_t are caller-owned and sized for max_seqs
 * sequences; the library allocates nothing. Host staging buffers should be
 * page-locked (cudaHostAlloc / cudaHostRegister) so the copies are
 * asynchronous. Per call, with n = number of sequences:
 *   q_host      [n][num_q_heads][head_dim]   (dtype)  query of each sequence
 *   k_new_host  [n][num_kv_heads][head_dim]  (dtype)  the appended token's K
 *   v_new_host  [n][num_kv_heads][head_dim]  (dtype)  ... and V
 *   out_host    [n][num_q_heads][head_dim]   (dtype)  attention output
 * Sequence i of seq_ids appends one token and is decoded with its new length.
 * If synchronize is non-zero the call returns after out_host holds the
 * result; otherwise the caller synchronises `stream` before reading it.
 * A block-manager failure (PA_ERR_NO_FREE_BLOCKS / PA_ERR_INVALID_ARG)
 * returns before anything is enqueued, state unchanged. A CUDA error after
 * the manager step leaves the manager with the step applied.
 *
 * Packed staging (optional): when the four small arrays are laid out back
 * to back on both sides, in the order slots [max_seqs] | pairs
 * [max_seqs][2] | context_lens [max_seqs] | tables [max_seqs][...], one
 * upload carries them (max_seqs * 28 + n * max_blocks_per_seq * 4 bytes);
 * pa_decode_step_h2d_bytes counts that copy.
 *
 * Pipelining (optional): with the fields at the end of the struct set
 * (pa_step_pipeline_create), the uploads run on `copy_stream` and the
 * download on `download_stream`:
 *   uploads   wait for download_done (this set's previous step has finished
 *             with its device staging), then record upload_done;
 *   kernels   on `stream` wait for upload_done, then record compute_done;
 *   download  waits for compute_done, then records download_done.
 * The host staging of a set is rewritten only after that set's previous
 * uploads completed (the call first waits on upload_done). A caller that
 * alternates two buffer sets with synchronize = 0 overlaps a step's uploads,
 * download and host work with the kernels of its neighbours. It keeps
 * q_host, k_new_host and v_new_host unchanged until the step's uploads are
 * done, and reads out_host after synchronising `download_stream`. Pool
 * updates stay ordered on `stream`. With the fields NULL everything runs on
 * `stream`.
 * ========================================================================= */
typedef struct {
  /* shape and cache */
  int max_seqs, num_q_heads, num_kv_heads, head_dim, block_size, num_blocks;
  int max_blocks_per_seq, partition_tokens;
  float scale;
  pa_dtype_t dtype;
  void* k_pool;
  void* v_pool;
  void* workspace;          /* pa_decode_split workspace (initialised) */
  size_t workspace_bytes;
  /* device staging */
  void* d_q;                /* [max_seqs][num_q_heads][head_dim] */
  void* d_k_new;            /* [max_seqs][num_kv_heads][head_dim] */
  void* d_v_new;
  void* d_out;              /* [max_seqs][num_q_heads][head_dim] */
  int64_t* d_slots;         /* [max_seqs] */
  int64_t* d_pairs;         /* [max_seqs][2] */
  int32_t* d_tables;        /* [max_seqs][max_blocks_per_seq] */
  int32_t* d_context_lens;  /* [max_seqs] */
  /* host staging (page-locked) */
  int64_t* h_slots;         /* [max_seqs] */
  int64_t* h_pairs;         /* [max_seqs][2] */
  int32_t* h_tables;        /* [max_seqs][max_blocks_per_seq] */
  int32_t* h_context_lens;  /* [max_seqs] */
  /* pipelining (optional, NULL = off; see above) */
  void* upload_done;        /* cudaEvent_t recorded on copy_stream after the uploads */
  void* compute_done;       /* cudaEvent_t recorded on `stream` after the decode */
  void* copy_stream;        /* cudaStream_t for the uploads */
  void* download_done;      /* cudaEvent_t recorded on download_stream after the download */
  void* download_stream;    /* cudaStream_t for the download */
} pa_step_buffers_t;

/* Creates the three events of a buffer set's pipelining fields (timing
 * disabled) and stores the two streams; the caller owns the streams.
 * pa_step_pipeline_destroy destroys the events and clears the fields.
 * Setup-time calls, not for the hot path. */
pa_status_t pa_step_pipeline_create(pa_step_buffers_t* buf, void* copy_stream,
                                    void* download_stream);
pa_status_t pa_step_pipeline_destroy(pa_step_buffers_t* buf);

/* Number of host->device and device->host bytes one pa_decode_step call of
 * n sequences moves when it makes `num_copies` copy-on-write copies. */
size_t pa_decode_step_h2d_bytes(const pa_step_buffers_t* buf, int n, int num_copies);
size_t pa_decode_step_d2h_bytes(const pa_step_buffers_t* buf, int n);

pa_status_t pa_decode_step(pa_bm_t bm, const pa_step_buffers_t* buf, const int64_t* seq_ids,
                           int n, const void* q_host, const void* k_new_host,
                           const void* v_new_host, void* out_host, int* num_copies,
                           int synchronize, uint32_t* dev_err, void* stream);

#ifdef __cplusplus
}  /* extern "C" */
#endif

#endif  /* PAGEDKV_H_ */
