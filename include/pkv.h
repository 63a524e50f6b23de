/*
 * pkv.h - exact attention over contiguous and paged K/V on B200 (sm_100a).
 *
 * A small C ABI: plain pointers and sizes, no C++ or framework types.
 *
 * What is computed, for every (batch or sequence, query head, query row):
 *
 *     O = softmax(Q K^T * scale) V
 *
 * exactly as defined in "Flash Attention: Fast, Memory-Efficient Attention for
 * LLMs", section "Standard Attention: The Memory Problem" (S = QK^T,
 * P = softmax(S), O = PV), but computed the way its section "The Algorithm"
 * describes: K/V are streamed in tiles, a running row maximum and running row
 * sum rescale an on-chip output accumulator, and S and P never reach global
 * memory.  Paged K/V are read in place through each sequence's block table
 * ("What is Paged FlashAttention?", sections "How does it work?" and
 * "Practical example"): token t of sequence s lives in physical page
 * block_table[s][t / page_size] at offset t % page_size, with no gather into a
 * contiguous copy first.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - Pointers named as device pointers must point to memory of the current CUDA
 *   device; the caller owns all memory.  Q/K/V/O, pages, tables and the
 *   workspace must be 16-byte aligned.  The library allocates nothing, frees
 *   nothing and never synchronises: all work is enqueued on `stream`
 *   (a cudaStream_t; NULL = the legacy default stream).
 * - Every function returns a pkv_status.  Argument errors are found on the
 *   host, before anything is launched, and nothing is launched then.  Launch
 *   failures return PKV_ERR_CUDA.  Errors that only the device can see
 *   (a page id outside [0, num_pages), a sequence length outside its table,
 *   a pipeline wait that ran out) never fault: the kernel skips the access,
 *   records a bit in a library-wide device error word and carries on;
 *   pkv_last_device_error() reads and clears it.  A page outside the pool is
 *   never read and its keys are left out of the softmax (decode and prefill
 *   alike), so that sequence gets attention over its other keys; a length
 *   outside its table is clamped into range.
 * - Masking: query row i (0-based, of q_len rows) may see key j (of kv_len keys)
 *   iff j <= i + (kv_len - q_len) when causal, every j < kv_len otherwise.
 *   With q_len == kv_len that is the lower triangle; with q_len == 1 (decode)
 *   every key is visible.
 * - Element types: PKV_BF16 (bfloat16 in and out, float32 accumulation, P
 *   rounded to bf16 before the PV product on the tensor-core path) and
 *   PKV_F32 (float32 in and out, float32 FMA throughout).
 * - Head dimension d: 128 for PKV_BF16; 64 or 128 for PKV_F32.
 * - Device reset: the library looks up, once per device, the device addresses
 *   of its own static arrays (the device error word; the scratch of
 *   paged_decode_noalloc) and keeps them for the life of the process.  A
 *   cudaDeviceReset, or anything else that destroys and re-creates a device's
 *   primary context, leaves those addresses stale: do not call the library on
 *   a device after resetting it in the same process.
 */
#ifndef PKV_H_
#define PKV_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define PKV_API __attribute__((visibility("default")))
#else
#define PKV_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  PKV_OK = 0,
  PKV_ERR_INVALID_ARG = 1,   /* a pointer, size, alignment or value is invalid */
  PKV_ERR_UNSUPPORTED = 2,   /* valid, but this build has no kernel for it (e.g. d = 96) */
  PKV_ERR_CUDA = 3,          /* a CUDA runtime call or launch failed */
  PKV_ERR_TIMEOUT = 4,       /* device: a pipeline wait gave up (pkv_last_device_error) */
  PKV_ERR_BAD_TABLE = 5,     /* device: a page id or sequence length was out of range */
  PKV_ERR_WORKSPACE = 6,     /* workspace missing or smaller than paged_attn_workspace_size() */
  PKV_ERR_OUT_OF_PAGES = 7   /* allocator: not enough free pages (nothing was changed) */
} pkv_status;

typedef enum { PKV_F32 = 0, PKV_BF16 = 1 } pkv_dtype;

/* Device error bits, as returned in *bits by pkv_last_device_error(). */
#define PKV_DEVERR_BAD_PAGE 0x1u   /* block_table entry outside [0, num_pages): its keys left out */
#define PKV_DEVERR_BAD_LEN 0x2u    /* seq_len outside [q_len, min(max_seq_len, pages*page_size)] */
#define PKV_DEVERR_TIMEOUT 0x4u    /* a bounded mbarrier wait ran out; the tile was abandoned */

/*
 * attn_prefill - attention over contiguous Q, K, V.
 *
 * Defines: "Flash Attention: Fast, Memory-Efficient Attention for LLMs",
 * sections "Standard Attention" (the operation) and "The Algorithm" (tiling
 * with online softmax; causal tiles past the diagonal are skipped, as its
 * "Flash Attention 2" section describes).
 *
 * Q, K, V, O : device pointers, [B, H, N, d] row-major (d contiguous), element
 *              type `dtype`.  O is written, nothing else is.
 * B, H, N, d : batch, heads, sequence length (queries = keys = N), head dim.
 *              B, H, N >= 1.
 * causal     : 0 or 1 (lower-triangular mask).
 * scale      : multiplier of QK^T, usually 1/sqrt(d); must be finite and > 0.
 * dtype      : PKV_BF16 (tcgen05 tensor-core kernel) or PKV_F32 (FMA kernel).
 * stream     : cudaStream_t the work is enqueued on.
 */
PKV_API int attn_prefill(const void* Q, const void* K, const void* V, void* O,
                 int B, int H, int N, int d, int causal, float scale,
                 int dtype, void* stream);

/*
 * pkv_test_prefill_stalled - test hook for the failure path; not for use in
 * production.
 *
 * The pages have no counterpart: it exists so that tests can make the bf16
 * prefill's bounded pipeline waits run out without faulting or hanging a GPU.
 * It runs what attn_prefill runs for dtype PKV_BF16 (same arguments, same
 * checks), except that every pipeline wait gives up after wait_limit_us
 * microseconds and the loader of each CTA's first work item never issues the
 * K load of K/V tile `stall_tile` (0-based).  Every CTA whose first item has
 * more than stall_tile K/V tiles then records PKV_DEVERR_TIMEOUT, stops,
 * drains the loads and MMAs it issued, frees its tensor memory and exits;
 * the output is undefined.  pkv_last_device_error() then returns
 * PKV_ERR_TIMEOUT, and later calls run normally.
 *
 * stall_tile    : >= 0.
 * wait_limit_us : in [1, 10^7].
 */
PKV_API int pkv_test_prefill_stalled(const void* Q, const void* K, const void* V, void* O,
                                     int B, int H, int N, int d, int causal, float scale,
                                     int stall_tile, int wait_limit_us, void* stream);

/*
 * attn_prefill_fp8qk - attention with e4m3 (FP8) Q and K, bf16 V and output.
 *
 * Defines: "Flash Attention: Fast, Memory-Efficient Attention for LLMs",
 * section "Flash Attention 3" (FP8 tensor cores for the QK^T product).  What
 * is computed, exactly as attn_prefill does it otherwise:
 *
 *     O = softmax((q_descale * Q8) (k_descale * K8)^T * scale) V
 *
 * where Q8, K8 hold e4m3 codes (1 sign, 4 exponent bits with bias 7, 3
 * mantissa bits; no infinities) and the descales are the per-tensor factors
 * the caller quantized with.  S = Q K^T runs on tcgen05 kind::f8f6f4; P and V
 * stay bf16 for the PV product.
 *
 * Q8, K8 : device, [B, H, N, d] e4m3 bytes.   V, O : device, [B, H, N, d] bf16.
 * d      : 128.  scale, q_descale, k_descale: finite and > 0.
 */
PKV_API int attn_prefill_fp8qk(const void* Q8, const void* K8, const void* V, void* O,
                               int B, int H, int N, int d, int causal, float scale,
                               float q_descale, float k_descale, void* stream);

/*
 * paged_attn_workspace_size - bytes of scratch paged_attn needs.
 *
 * Decode (q_len == 1) splits each sequence's keys into fixed-size chunks that
 * run in parallel and are merged with a log-sum-exp combine; the partial
 * (O, max, sum) of every chunk lives in this workspace.  The size depends only
 * on these arguments (same arguments, same plan).  Returns 0 when one chunk
 * per sequence suffices (no workspace needed), and 0 for invalid arguments.
 */
PKV_API size_t paged_attn_workspace_size(int num_seqs, int H, int d, int max_seq_len, int page_size);

/*
 * paged_attn - attention of new query tokens against a paged K/V cache.
 *
 * Defines: "What is Paged FlashAttention?", sections "How does it work?"
 * (locate pages through the block table, load K/V tiles, online softmax,
 * accumulate without a full-cache gather) and "Practical example" (logical
 * page t / page_size, offset t % page_size, physical page
 * block_table[logical]).  Pages follow "FlashAttention and PagedAttention:
 * Two Fixes for Two Different Bottlenecks", section "PagedAttention ... How
 * it works": fixed-size blocks, a per-sequence block table, blocks may be
 * shared by several sequences (pages are only read here).
 *
 * q           : device, [num_seqs, H, q_len, d]; the q_len newest tokens of each
 *               sequence (their K/V are already in the cache).
 * k_pages,
 * v_pages     : device, [num_pages, page_size, H_kv, d].
 * block_table : device int32, [num_seqs, max_pages_per_seq]; entries past
 *               ceil(seq_lens[s] / page_size) are never read (pad with -1).
 * seq_lens    : device int32, [num_seqs]; kv length of each sequence, the q_len
 *               new tokens included.  Must satisfy
 *               q_len <= seq_lens[s] <= min(max_seq_len, max_pages_per_seq * page_size).
 * page_size   : tokens per page, a power of two in [16, 256].
 * q_len       : 1 = decode (split-K kernel); > 1 = paged prefill (tensor-core
 *               kernel for PKV_BF16, FMA kernel for PKV_F32).
 * H, H_kv     : query heads and kv heads; H % H_kv == 0 (query head h reads
 *               kv head h / (H / H_kv)).
 * num_pages   : pages in the pool (page ids must be < num_pages).
 * max_seq_len : host-known upper bound of seq_lens (plans the split-K grid).
 * out         : device, [num_seqs, H, q_len, d], element type `dtype`.
 * workspace   : device scratch of >= paged_attn_workspace_size(num_seqs, H, d,
 *               max_seq_len, page_size) bytes, 256-byte aligned (NULL if that
 *               size is 0).  Its contents need no initialisation and are
 *               garbage afterwards.  Two calls in flight at once need two
 *               workspaces.
 *
 * Launches (all on `stream`): q_len == 1 enqueues the split kernel and, when
 * some sequence spans more than one split, a merge kernel after it.  With
 * H > H_kv the merge is a programmatic dependent launch: it may be scheduled
 * while the split kernel drains, and it waits on the device for that kernel's
 * results, so stream order is kept (also under stream capture).
 */
PKV_API int paged_attn(const void* q, const void* k_pages, const void* v_pages,
               const int32_t* block_table, const int32_t* seq_lens,
               int page_size, int num_seqs, int q_len, int H, int H_kv, int d,
               int num_pages, int max_pages_per_seq, int max_seq_len,
               int causal, float scale, int dtype,
               void* out, void* workspace, size_t workspace_bytes, void* stream);

/*
 * paged_decode_noalloc - paged decode that allocates nothing and needs no
 * workspace argument.
 *
 * The pages have no counterpart for this entry point; it exists for callers
 * that cannot allocate device memory where they call attention: a plugin
 * invoked from another runtime's enqueue hook that offers no allocator, a
 * latency-critical loop in which cudaMalloc/cudaFree would synchronise the
 * device, or a process whose device memory a pool has reserved in full.
 *
 * It computes what paged_attn computes for q_len == 1 and PKV_BF16 (decode:
 * every cached key is visible), with the same kernels and split plan, and the
 * same meaning, layout and validation of the arguments paged_attn shares with
 * it (d must be 128).  The split partials live in a static device array of
 * PKV_NOALLOC_SCRATCH_BYTES inside the library: every GPU that loads the
 * library holds that memory until the process exits.
 *
 * - Limit: when paged_attn_workspace_size(num_seqs, H, d, max_seq_len,
 *   page_size) exceeds PKV_NOALLOC_SCRATCH_BYTES the call returns
 *   PKV_ERR_WORKSPACE and launches nothing.
 * - Set-up: the first call on each device looks up the array's device address
 *   (cudaGetSymbolAddress, with that device current) and caches it for the
 *   life of the process (so not across a device reset, see above); make that
 *   first call before any stream capture.
 * - Sharing: all calls on a device use the same array, which keeps the last
 *   call's contents.  No part of it needs to start at zero (a call writes every
 *   partial it reads), but calls whose kernels overlap on the GPU (other
 *   streams, other host threads) race on it: serialise them.
 */
#define PKV_NOALLOC_SCRATCH_BYTES (64u << 20)
PKV_API int paged_decode_noalloc(const void* q, const void* k_pages, const void* v_pages,
                                 const int32_t* block_table, const int32_t* seq_lens,
                                 int page_size, int num_seqs, int H, int H_kv, int d,
                                 int num_pages, int max_pages_per_seq, int max_seq_len,
                                 float scale, void* out, void* stream);

/* ------------------------------------------------------------------------ */
/* The write side of the paged cache.                                       */
/* ------------------------------------------------------------------------ */

/*
 * paged_kv_append - write new tokens' K and V rows into their pages.
 *
 * Defines: "Flash Attention: Fast, Memory-Efficient Attention for LLMs",
 * section "KV Cache" (each decode step appends the new K_t, V_t; prefill
 * stores the K/V of every prompt token), with the address of token position
 * pos of sequence s given by "What is Paged FlashAttention?", "Practical
 * example": page block_table[s][pos / page_size], offset pos % page_size.
 *
 * k_new, v_new : device, [num_new, H_kv, d]: rows of all sequences' new tokens,
 *                sequence by sequence.
 * cu_new       : device int32 [num_seqs + 1], non-decreasing, cu_new[0] = 0,
 *                cu_new[num_seqs] = num_new: sequence s owns rows
 *                [cu_new[s], cu_new[s+1]).
 * start_pos    : device int32 [num_seqs]: position of sequence s's first new
 *                token (its length before the append).
 * block_table  : device int32 [num_seqs, max_pages_per_seq]; the pages covering
 *                the new positions must already be allocated (pkv_alloc_reserve).
 * k_pages,
 * v_pages      : device, [num_pages, page_size, H_kv, d], written in place.
 * dtype        : PKV_BF16 or PKV_F32; d is 64 or 128.
 * A row whose page id is outside [0, num_pages) or whose position is past the
 * table is skipped and flagged (PKV_DEVERR_BAD_PAGE / PKV_DEVERR_BAD_LEN).
 * Rows must not target the same slot twice in one call.
 * Returns PKV_OK without reading any pointer or launching when num_new == 0;
 * PKV_ERR_INVALID_ARG for a negative num_new, num_seqs, max_pages_per_seq,
 * num_pages or H_kv below 1, a page_size that is not a power of two in
 * [16, 256], an unknown dtype, or a null or misaligned pointer (16 bytes for
 * row data, 4 for the int32 arrays); PKV_ERR_UNSUPPORTED for d other than 64
 * or 128, or a pool of more than 2^31 token rows.
 */
PKV_API int paged_kv_append(const void* k_new, const void* v_new, const int32_t* cu_new,
                            const int32_t* start_pos, const int32_t* block_table,
                            int max_pages_per_seq, int num_seqs, int num_new, void* k_pages,
                            void* v_pages, int num_pages, int page_size, int H_kv, int d,
                            int dtype, void* stream);

/*
 * paged_kv_copy_pages - copy whole pages (K and V): page src[i] -> page dst[i].
 *
 * Defines the copy half of copy-on-write ("FlashAttention and PagedAttention:
 * Two Fixes for Two Different Bottlenecks", section "PagedAttention ... How it
 * works": sequences share prefix blocks and copy only when they diverge).
 * src, dst : device int32 [n]; ids in [0, num_pages) (others are skipped and
 *            flagged); a dst must not also be a src in the same call.
 * Returns PKV_OK without reading any pointer or launching when n == 0;
 * PKV_ERR_INVALID_ARG for a negative n, num_pages or H_kv below 1, a page_size
 * that is not a power of two in [16, 256], an unknown dtype, or a null or
 * misaligned pointer (16 bytes for the pools, 4 for src and dst);
 * PKV_ERR_UNSUPPORTED for d other than 64 or 128.
 */
PKV_API int paged_kv_copy_pages(void* k_pages, void* v_pages, const int32_t* src,
                                const int32_t* dst, int n, int num_pages, int page_size,
                                int H_kv, int d, int dtype, void* stream);

/*
 * pkv_alloc_* - host page allocator (bookkeeping only; host memory).
 *
 * Defines: "FlashAttention and PagedAttention: Two Fixes for Two Different
 * Bottlenecks", section "PagedAttention ... How it works" (fixed-size blocks,
 * per-sequence block table, allocation on demand, shared prefixes with
 * copy-on-write) and "Flash Attention: Fast, Memory-Efficient Attention for
 * LLMs", section "PagedAttention (vLLM)" (pages of finished sequences are
 * freed and reused).  Policy: the smallest free page id is handed out first;
 * pages carry reference counts; only a shared, partially filled last page is
 * ever copied, just before the sequence writes into it.  Not thread-safe.
 *
 * pkv_alloc_create    : pool of num_pages pages of page_size tokens; tables
 *                       hold at most max_pages_per_seq pages.  NULL on error.
 * pkv_alloc_add_seq   : register an empty sequence under seq_id.
 * pkv_alloc_reserve   : grow seq_id by n_tokens.  *start_pos gets the position
 *                       of its first new token.  If its partially filled last
 *                       page is shared, that page is replaced by a fresh one
 *                       and the copy the caller must run first (with
 *                       paged_kv_copy_pages) is returned in *cow_src ->
 *                       *cow_dst with *n_cow = 1 (else *n_cow = 0).
 *                       PKV_ERR_OUT_OF_PAGES leaves everything unchanged.
 * pkv_alloc_fork      : child_id shares all of parent_id's pages (same length).
 * pkv_alloc_free_seq  : drop seq_id; pages nobody else holds return to the pool.
 * pkv_alloc_seq_len   : current length of seq_id.
 * pkv_alloc_block_table: host arrays table [n][max_pages_per_seq] (-1 padded)
 *                       and seq_lens [n] for the n listed sequences.
 * pkv_alloc_num_free  : free pages (-1 for NULL).
 * pkv_alloc_page_refs : reference count of a page (-1 if out of range).
 */
typedef struct pkv_allocator pkv_allocator;
PKV_API pkv_allocator* pkv_alloc_create(int num_pages, int page_size, int max_pages_per_seq);
PKV_API void pkv_alloc_destroy(pkv_allocator* a);
PKV_API int pkv_alloc_add_seq(pkv_allocator* a, int seq_id);
PKV_API int pkv_alloc_reserve(pkv_allocator* a, int seq_id, int n_tokens, int32_t* start_pos,
                              int32_t* cow_src, int32_t* cow_dst, int* n_cow);
PKV_API int pkv_alloc_fork(pkv_allocator* a, int parent_id, int child_id);
PKV_API int pkv_alloc_free_seq(pkv_allocator* a, int seq_id);
PKV_API int pkv_alloc_seq_len(const pkv_allocator* a, int seq_id, int* len);
PKV_API int pkv_alloc_block_table(const pkv_allocator* a, const int* seq_ids, int n,
                                  int32_t* table, int32_t* seq_lens);
PKV_API int pkv_alloc_num_free(const pkv_allocator* a);
PKV_API int pkv_alloc_page_refs(const pkv_allocator* a, int page);

/*
 * pkv_resolve - host-side page-table address resolution (for tests and tools).
 *
 * Defines: "What is Paged FlashAttention?", section "Practical example".
 * block_table_row : host int32 array of n_entries page ids.
 * token           : 0-based token index; must be < n_entries * page_size.
 * phys, offset    : host outputs: block_table_row[token / page_size] and
 *                   token % page_size.  (page_size 256, row [5,1,9], token 300
 *                   -> phys 1, offset 44.)
 */
PKV_API int pkv_resolve(const int32_t* block_table_row, int n_entries, int page_size,
                int token, int32_t* phys, int32_t* offset);

/*
 * pkv_last_device_error - read and clear the device error word.
 *
 * Synchronises `stream`, then returns PKV_ERR_TIMEOUT if a wait gave up,
 * PKV_ERR_BAD_TABLE if a page id or length was out of range, PKV_OK otherwise.
 * `bits` (host, may be NULL) receives the raw PKV_DEVERR_* bits.  The word is
 * per device and shared by every call on it.
 */
PKV_API int pkv_last_device_error(void* stream, unsigned int* bits);

/* pkv_status_string - static, NUL-terminated description of a status code. */
PKV_API const char* pkv_status_string(int status);

#ifdef __cplusplus
}
#endif

#endif /* PKV_H_ */
