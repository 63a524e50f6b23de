// The write side of the paged KV cache: appending new tokens' K/V rows into
// their pages, and copying whole pages (copy-on-write of a shared last page).
//
// "Flash Attention: Fast, Memory-Efficient Attention for LLMs", section "KV
// Cache": each decode step appends the new token's K_t, V_t to the cache;
// prefill writes the K/V of all prompt tokens.  Where a row lands is the page
// table lookup of "What is Paged FlashAttention?", "Practical example":
// page block_table[s][pos / page_size], offset pos % page_size.
//
// Both kernels are plain copies bound by HBM: one CTA per token row (all H_kv
// heads of a token are contiguous in a page, [page][offset][H_kv][d]), 16-byte
// vector loads and stores, every byte read once and written once.
#include "common.cuh"

namespace pkv {
namespace {

constexpr int kThreads = 128;

__global__ void __launch_bounds__(kThreads) append_kernel(const AppendParams p) {
  const int i = blockIdx.x;                       // new-token row
  __shared__ int s_dst;                            // destination token row in the pool, or -1
  if (threadIdx.x == 0) {
    // sequence of row i: the last s with cu_new[s] <= i (binary search)
    int lo = 0, hi = p.num_seqs - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (p.cu_new[mid] <= i) lo = mid; else hi = mid - 1;
    }
    const int s = lo;
    const int pos = p.start_pos[s] + (i - p.cu_new[s]);
    const int lp = pos >> p.page_shift;
    int dst = -1;
    if (pos < 0 || lp >= p.max_pages) {
      flag_error(p.err, PKV_DEVERR_BAD_LEN);
    } else {
      const int phys = p.block_table[(size_t)s * p.max_pages + lp];
      if (phys < 0 || phys >= p.num_pages)
        flag_error(p.err, PKV_DEVERR_BAD_PAGE);
      else
        dst = phys * p.page_size + (pos & (p.page_size - 1));
    }
    s_dst = dst;
  }
  __syncthreads();
  const int dst = s_dst;
  if (dst < 0) return;
  const size_t vec = p.row_bytes / 16;
  const uint4* ks = reinterpret_cast<const uint4*>(static_cast<const char*>(p.k_new) + (size_t)i * p.row_bytes);
  const uint4* vs = reinterpret_cast<const uint4*>(static_cast<const char*>(p.v_new) + (size_t)i * p.row_bytes);
  uint4* kd = reinterpret_cast<uint4*>(static_cast<char*>(p.k_pages) + (size_t)dst * p.row_bytes);
  uint4* vd = reinterpret_cast<uint4*>(static_cast<char*>(p.v_pages) + (size_t)dst * p.row_bytes);
  for (size_t v = threadIdx.x; v < vec; v += kThreads) {
    const uint4 a = ldg_nc_v4(ks + v);
    const uint4 b = ldg_nc_v4(vs + v);
    kd[v] = a;
    vd[v] = b;
  }
}

// grid = (pairs, chunks of a page); copies page src[i] -> dst[i] in K and V.
__global__ void __launch_bounds__(kThreads) copy_pages_kernel(const CopyPagesParams p) {
  const int i = blockIdx.x;
  const int src = p.src[i], dst = p.dst[i];
  if (src < 0 || src >= p.num_pages || dst < 0 || dst >= p.num_pages) {
    if (blockIdx.y == 0 && threadIdx.x == 0) flag_error(p.err, PKV_DEVERR_BAD_PAGE);
    return;
  }
  const size_t vec = p.page_bytes / 16;
  const size_t per = (vec + gridDim.y - 1) / gridDim.y;
  const size_t v0 = blockIdx.y * per, v1 = min(vec, v0 + per);
  const uint4* ks = reinterpret_cast<const uint4*>(static_cast<const char*>(p.k_pages) + (size_t)src * p.page_bytes);
  const uint4* vs = reinterpret_cast<const uint4*>(static_cast<const char*>(p.v_pages) + (size_t)src * p.page_bytes);
  uint4* kd = reinterpret_cast<uint4*>(static_cast<char*>(p.k_pages) + (size_t)dst * p.page_bytes);
  uint4* vd = reinterpret_cast<uint4*>(static_cast<char*>(p.v_pages) + (size_t)dst * p.page_bytes);
  for (size_t v = v0 + threadIdx.x; v < v1; v += kThreads) {
    kd[v] = ks[v];
    vd[v] = vs[v];
  }
}

}  // namespace

cudaError_t launch_append(const AppendParams& p, cudaStream_t stream) {
  if (p.num_new == 0) return cudaSuccess;
  append_kernel<<<p.num_new, kThreads, 0, stream>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_copy_pages(const CopyPagesParams& p, cudaStream_t stream) {
  if (p.n == 0) return cudaSuccess;
  const size_t vec = p.page_bytes / 16;
  unsigned chunks = (unsigned)((vec + kThreads * 8 - 1) / (kThreads * 8));   // ~16 KB per CTA
  chunks = chunks < 1 ? 1 : (chunks > 65535 ? 65535 : chunks);
  copy_pages_kernel<<<dim3(p.n, chunks), kThreads, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace pkv
