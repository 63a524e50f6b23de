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
 *   pkv_last_device_error() reads and clears it.
 * - Masking: query row i (0-based, of q_len rows) may see key j (of kv_len keys)
 *   iff j <= i + (kv_len - q_len) when causal, every j < kv_len otherwise.
 *   With q_len == kv_len that is the lower triangle; with q_len == 1 (decode)
 *   every key is visible.
 * - Element types: PKV_BF16 (bfloat16 in and out, float32 accumulation, P
 *   rounded to bf16 before the PV product on the tensor-core path) and
 *   PKV_F32 (float32 in and out, float32 FMA throughout).
 * - Head dimension d: 128 for PKV_BF16; 64 or 128 for PKV_F32.
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
  PKV_ERR_WORKSPACE = 6      /* workspace missing or smaller than paged_attn_workspace_size() */
} pkv_status;

typedef enum { PKV_F32 = 0, PKV_BF16 = 1 } pkv_dtype;

/* Device error bits, as returned in *bits by pkv_last_device_error(). */
#define PKV_DEVERR_BAD_PAGE 0x1u   /* block_table entry outside [0, num_pages): page skipped */
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
 *   (cudaGetSymbolAddress, with that device current) and caches it; make that
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
