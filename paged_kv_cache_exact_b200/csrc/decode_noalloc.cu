// Allocation-free paged decode: the split-K decode kernel with its scratch in
// a static device array owned by this library instead of a caller workspace.
//
// Who needs it: code that must not allocate device memory at the point where
// it calls attention -- a plugin called from another runtime's enqueue hook
// that hands out no allocator, a latency-critical serving loop where
// cudaMalloc/cudaFree would synchronise the device, or a process whose device
// memory is fully reserved up front by a pool.  Such callers pass only their
// inputs and outputs; the split partials live in `g_decode_scratch`.
//
// Cost of the design: every GPU that loads libpkv.so holds
// PKV_NOALLOC_SCRATCH_BYTES of device memory until the process exits, and all
// calls on a device share that one array.
#include <mutex>

#include "common.cuh"

namespace {

// Split partials (unnormalised O, then (max, sum) pairs), reused by every call.
static __device__ __align__(256) unsigned char g_decode_scratch[PKV_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
void* g_scratch_ptr[kMaxDevices] = {};
std::mutex g_scratch_mu;

// Device address of the scratch array on the current device.  In host code
// `g_decode_scratch` names a host-side stand-in, not device memory, so the
// address is looked up once per device (with that device current) and cached.
int scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return PKV_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || !p) return PKV_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return PKV_OK;
}

bool aligned16(const void* p) { return p && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void* p) { return p && (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

}  // namespace

extern "C" PKV_API int paged_decode_noalloc(const void* q, const void* k_pages,
                                            const void* v_pages, const int32_t* block_table,
                                            const int32_t* seq_lens, int page_size, int num_seqs,
                                            int H, int H_kv, int d, int num_pages,
                                            int max_pages_per_seq, int max_seq_len, float scale,
                                            void* out, void* stream) {
  if (!aligned16(q) || !aligned16(k_pages) || !aligned16(v_pages) || !aligned16(out) ||
      !aligned4(block_table) || !aligned4(seq_lens))
    return PKV_ERR_INVALID_ARG;
  if (page_size < 16 || page_size > 256 || (page_size & (page_size - 1))) return PKV_ERR_INVALID_ARG;
  if (num_seqs < 1 || H < 1 || H_kv < 1 || H % H_kv != 0 || num_pages < 1 ||
      max_pages_per_seq < 1 || max_seq_len < 1 || !(scale > 0.f) || scale == INFINITY)
    return PKV_ERR_INVALID_ARG;
  if ((long long)max_pages_per_seq * page_size < max_seq_len) return PKV_ERR_INVALID_ARG;
  if (d != 128) return PKV_ERR_UNSUPPORTED;
  if (num_seqs > 65535 || H > 65535 || (long long)num_pages * page_size > (1LL << 31))
    return PKV_ERR_UNSUPPORTED;

  int split = 0, nsplit = 0;
  pkv::decode_plan(num_seqs, H, max_seq_len, page_size, &split, &nsplit);
  if (split / page_size > 256) return PKV_ERR_UNSUPPORTED;
  // Same layout as the caller-workspace path: partial O, then (max, sum) pairs.
  const size_t per = (size_t)num_seqs * H * nsplit;
  const size_t o_bytes = (per * d * sizeof(float) + 255) & ~size_t(255);
  const size_t need = nsplit > 1 ? o_bytes + per * sizeof(float2) : 0;
  if (need > PKV_NOALLOC_SCRATCH_BYTES) return PKV_ERR_WORKSPACE;   // beyond the fixed maximum

  void* scratch = nullptr;
  if (int r = scratch_address(&scratch)) return r;
  unsigned int* err = nullptr;
  if (int r = pkv::device_error_word(&err)) return r;

  pkv::DecodeParams p{};
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.k_pages = static_cast<const __nv_bfloat16*>(k_pages);
  p.v_pages = static_cast<const __nv_bfloat16*>(v_pages);
  p.block_table = block_table, p.seq_lens = seq_lens;
  p.out = static_cast<__nv_bfloat16*>(out);
  if (need > 0) {
    // Nothing here needs clearing: each call writes every partial it later reads.
    p.ws_o = static_cast<float*>(scratch);
    p.ws_ml = reinterpret_cast<float2*>(static_cast<char*>(scratch) + o_bytes);
  }
  p.err = err;
  p.num_seqs = num_seqs, p.H = H, p.H_kv = H_kv;
  p.page_size = page_size;
  int shift = 0;
  while ((1 << shift) < page_size) ++shift;
  p.page_shift = shift;
  p.num_pages = num_pages, p.max_pages = max_pages_per_seq, p.max_seq_len = max_seq_len;
  p.split_tokens = split, p.max_splits = nsplit;
  p.scale_log2 = scale * pkv::kLog2e;
  return pkv::cuda_status(pkv::launch_decode_bf16(p, static_cast<cudaStream_t>(stream)));
}
