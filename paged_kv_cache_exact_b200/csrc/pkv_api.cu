// The C ABI declared in include/pkv.h: host-side validation, planning and
// dispatch to the kernels.  Nothing here allocates device memory or
// synchronises, except pkv_last_device_error (documented to synchronise).
#include <cmath>
#include <mutex>

#include "common.cuh"

// Library-wide device error word (PKV_DEVERR_* bits), one per device.
static __device__ unsigned int g_pkv_error_word;

namespace {

constexpr int kMaxDevices = 64;
unsigned int* g_err_ptr[kMaxDevices] = {};
std::mutex g_err_mu;

// Device address of the error word on the current device (looked up once).
int error_word(unsigned int** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return PKV_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_err_mu);
  if (!g_err_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_pkv_error_word) != cudaSuccess) return PKV_ERR_CUDA;
    g_err_ptr[dev] = static_cast<unsigned int*>(p);
  }
  *out = g_err_ptr[dev];
  return PKV_OK;
}

bool aligned16(const void* p) { return p && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void* p) { return p && (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }
bool pow2(int x) { return x > 0 && (x & (x - 1)) == 0; }
int log2i(int x) {
  int s = 0;
  while ((1 << s) < x) ++s;
  return s;
}
bool good_scale(float s) { return std::isfinite(s) && s > 0.f; }

}  // namespace

namespace pkv {
int device_error_word(unsigned int** out) { return error_word(out); }
int cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return PKV_OK;
  if (e == cudaErrorNotSupported) return PKV_ERR_UNSUPPORTED;
  return PKV_ERR_CUDA;
}
}  // namespace pkv

using pkv::cuda_status;

extern "C" {

const char* pkv_status_string(int status) {
  switch (status) {
    case PKV_OK: return "ok";
    case PKV_ERR_INVALID_ARG: return "invalid argument";
    case PKV_ERR_UNSUPPORTED: return "unsupported configuration";
    case PKV_ERR_CUDA: return "CUDA runtime or launch error";
    case PKV_ERR_TIMEOUT: return "device pipeline wait timed out";
    case PKV_ERR_BAD_TABLE: return "page id or sequence length out of range";
    case PKV_ERR_WORKSPACE: return "workspace missing or too small";
    case PKV_ERR_OUT_OF_PAGES: return "no free pages left in the pool";
    default: return "unknown status";
  }
}

int pkv_resolve(const int32_t* block_table_row, int n_entries, int page_size, int token,
                int32_t* phys, int32_t* offset) {
  if (!block_table_row || !phys || !offset || n_entries <= 0 || page_size <= 0 || token < 0)
    return PKV_ERR_INVALID_ARG;
  const long long logical = token / page_size;
  if (logical >= n_entries) return PKV_ERR_INVALID_ARG;
  *phys = block_table_row[logical];
  *offset = token % page_size;
  return PKV_OK;
}

int attn_prefill(const void* Q, const void* K, const void* V, void* O, int B, int H, int N,
                 int d, int causal, float scale, int dtype, void* stream) {
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O)) return PKV_ERR_INVALID_ARG;
  if (B < 1 || H < 1 || N < 1 || (causal != 0 && causal != 1) || !good_scale(scale))
    return PKV_ERR_INVALID_ARG;
  if (B > 65535 || H > 65535) return PKV_ERR_UNSUPPORTED;
  unsigned int* err = nullptr;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (dtype == PKV_F32) {
    if (d != 64 && d != 128) return PKV_ERR_UNSUPPORTED;
    if (int r = error_word(&err)) return r;
    pkv::SimtParams p{};
    p.q = static_cast<const float*>(Q);
    p.k = static_cast<const float*>(K);
    p.v = static_cast<const float*>(V);
    p.out = static_cast<float*>(O);
    p.err = err;
    p.B = B, p.H = H, p.H_kv = H, p.q_len = N, p.kv_len = N, p.d = d;
    p.paged = 0, p.causal = causal;
    p.scale_log2 = scale * pkv::kLog2e;
    return cuda_status(pkv::launch_simt_f32(p, st));
  }
  if (dtype == PKV_BF16) {
    if (d != 128) return PKV_ERR_UNSUPPORTED;
    if (int r = error_word(&err)) return r;
    pkv::PrefillParams p{};
    p.Q = Q, p.K = K, p.V = V, p.O = O;
    p.err = err;
    p.B = B, p.H = H, p.H_kv = H, p.q_len = N, p.kv_len = N, p.d = d;
    p.paged = 0, p.causal = causal;
    p.scale_log2 = scale * pkv::kLog2e;
    return cuda_status(pkv::launch_prefill_bf16(p, st));
  }
  return PKV_ERR_INVALID_ARG;
}

int pkv_test_prefill_stalled(const void* Q, const void* K, const void* V, void* O, int B, int H,
                             int N, int d, int causal, float scale, int stall_tile,
                             int wait_limit_us, void* stream) {
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O)) return PKV_ERR_INVALID_ARG;
  if (B < 1 || H < 1 || N < 1 || (causal != 0 && causal != 1) || !good_scale(scale) ||
      stall_tile < 0 || wait_limit_us < 1 || wait_limit_us > 10000000)
    return PKV_ERR_INVALID_ARG;
  if (d != 128 || B > 65535 || H > 65535) return PKV_ERR_UNSUPPORTED;
  unsigned int* err = nullptr;
  if (int r = error_word(&err)) return r;
  pkv::PrefillParams p{};
  p.Q = Q, p.K = K, p.V = V, p.O = O;
  p.err = err;
  p.B = B, p.H = H, p.H_kv = H, p.q_len = N, p.kv_len = N, p.d = d;
  p.paged = 0, p.causal = causal;
  p.scale_log2 = scale * pkv::kLog2e;
  p.wait_limit_ns = 1000ull * (unsigned long long)wait_limit_us;
  p.stall_tile_plus1 = stall_tile + 1;
  return cuda_status(pkv::launch_prefill_bf16(p, static_cast<cudaStream_t>(stream)));
}

int attn_prefill_fp8qk(const void* Q8, const void* K8, const void* V, void* O, int B, int H,
                       int N, int d, int causal, float scale, float q_descale, float k_descale,
                       void* stream) {
  if (!aligned16(Q8) || !aligned16(K8) || !aligned16(V) || !aligned16(O)) return PKV_ERR_INVALID_ARG;
  if (B < 1 || H < 1 || N < 1 || (causal != 0 && causal != 1) || !good_scale(scale) ||
      !good_scale(q_descale) || !good_scale(k_descale))
    return PKV_ERR_INVALID_ARG;
  if (d != 128) return PKV_ERR_UNSUPPORTED;
  if (B > 65535 || H > 65535) return PKV_ERR_UNSUPPORTED;
  unsigned int* err = nullptr;
  if (int r = error_word(&err)) return r;
  pkv::PrefillParams p{};
  p.Q = Q8, p.K = K8, p.V = V, p.O = O;
  p.err = err;
  p.B = B, p.H = H, p.H_kv = H, p.q_len = N, p.kv_len = N, p.d = d;
  p.paged = 0, p.causal = causal, p.fp8_qk = 1;
  p.scale_log2 = scale * q_descale * k_descale * pkv::kLog2e;
  return cuda_status(pkv::launch_prefill_bf16(p, static_cast<cudaStream_t>(stream)));
}

size_t paged_attn_workspace_size(int num_seqs, int H, int d, int max_seq_len, int page_size) {
  if (num_seqs < 1 || H < 1 || d < 1 || max_seq_len < 1 || !pow2(page_size)) return 0;
  int split = 0, nsplit = 0;
  pkv::decode_plan(num_seqs, H, max_seq_len, page_size, &split, &nsplit);
  if (nsplit <= 1) return 0;
  const size_t per = (size_t)num_seqs * H * nsplit;
  size_t o_bytes = per * d * sizeof(float);
  o_bytes = (o_bytes + 255) & ~size_t(255);
  return o_bytes + per * sizeof(float2);
}

int paged_attn(const void* q, const void* k_pages, const void* v_pages,
               const int32_t* block_table, const int32_t* seq_lens, int page_size,
               int num_seqs, int q_len, int H, int H_kv, int d, int num_pages,
               int max_pages_per_seq, int max_seq_len, int causal, float scale, int dtype,
               void* out, void* workspace, size_t workspace_bytes, void* stream) {
  if (!aligned16(q) || !aligned16(k_pages) || !aligned16(v_pages) || !aligned16(out) ||
      !aligned4(block_table) || !aligned4(seq_lens))
    return PKV_ERR_INVALID_ARG;
  if (!pow2(page_size) || page_size < 16 || page_size > 256) return PKV_ERR_INVALID_ARG;
  if (num_seqs < 1 || q_len < 1 || H < 1 || H_kv < 1 || H % H_kv != 0 || num_pages < 1 ||
      max_pages_per_seq < 1 || max_seq_len < q_len || (causal != 0 && causal != 1) ||
      !good_scale(scale))
    return PKV_ERR_INVALID_ARG;
  if ((long long)max_pages_per_seq * page_size < max_seq_len) return PKV_ERR_INVALID_ARG;
  if (num_seqs > 65535 || H > 65535 || (long long)num_pages * page_size > (1LL << 31))
    return PKV_ERR_UNSUPPORTED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  unsigned int* err = nullptr;

  if (dtype == PKV_F32) {
    if (d != 64 && d != 128) return PKV_ERR_UNSUPPORTED;
    if (int r = error_word(&err)) return r;
    pkv::SimtParams p{};
    p.q = static_cast<const float*>(q);
    p.k = static_cast<const float*>(k_pages);
    p.v = static_cast<const float*>(v_pages);
    p.block_table = block_table, p.seq_lens = seq_lens;
    p.out = static_cast<float*>(out);
    p.err = err;
    p.B = num_seqs, p.H = H, p.H_kv = H_kv, p.q_len = q_len, p.kv_len = 0, p.d = d;
    p.paged = 1, p.page_size = page_size, p.page_shift = log2i(page_size);
    p.num_pages = num_pages, p.max_pages = max_pages_per_seq, p.max_seq_len = max_seq_len;
    p.causal = causal;
    p.scale_log2 = scale * pkv::kLog2e;
    return cuda_status(pkv::launch_simt_f32(p, st));
  }
  if (dtype != PKV_BF16) return PKV_ERR_INVALID_ARG;
  if (d != 128) return PKV_ERR_UNSUPPORTED;

  if (q_len == 1) {
    int split = 0, nsplit = 0;
    pkv::decode_plan(num_seqs, H, max_seq_len, page_size, &split, &nsplit);
    if (split / page_size > 256) return PKV_ERR_UNSUPPORTED;
    const size_t need = paged_attn_workspace_size(num_seqs, H, d, max_seq_len, page_size);
    if (need > 0 && (!workspace || workspace_bytes < need ||
                     (reinterpret_cast<uintptr_t>(workspace) & 255u)))
      return PKV_ERR_WORKSPACE;
    if (int r = error_word(&err)) return r;
    pkv::DecodeParams p{};
    p.q = static_cast<const __nv_bfloat16*>(q);
    p.k_pages = static_cast<const __nv_bfloat16*>(k_pages);
    p.v_pages = static_cast<const __nv_bfloat16*>(v_pages);
    p.block_table = block_table, p.seq_lens = seq_lens;
    p.out = static_cast<__nv_bfloat16*>(out);
    if (need > 0) {
      const size_t per = (size_t)num_seqs * H * nsplit;
      size_t o_bytes = (per * d * sizeof(float) + 255) & ~size_t(255);
      p.ws_o = static_cast<float*>(workspace);
      p.ws_ml = reinterpret_cast<float2*>(static_cast<char*>(workspace) + o_bytes);
    }
    p.err = err;
    p.num_seqs = num_seqs, p.H = H, p.H_kv = H_kv;
    p.page_size = page_size, p.page_shift = log2i(page_size);
    p.num_pages = num_pages, p.max_pages = max_pages_per_seq, p.max_seq_len = max_seq_len;
    p.split_tokens = split, p.max_splits = nsplit;
    p.scale_log2 = scale * pkv::kLog2e;
    return cuda_status(pkv::launch_decode_bf16(p, st));
  }

  if (int r = error_word(&err)) return r;
  pkv::PrefillParams p{};
  p.Q = q, p.K = k_pages, p.V = v_pages, p.O = out;
  p.block_table = block_table, p.seq_lens = seq_lens;
  p.err = err;
  p.B = num_seqs, p.H = H, p.H_kv = H_kv, p.q_len = q_len, p.kv_len = 0, p.d = d;
  p.paged = 1, p.page_size = page_size, p.page_shift = log2i(page_size);
  p.num_pages = num_pages, p.max_pages = max_pages_per_seq, p.max_seq_len = max_seq_len;
  p.causal = causal;
  p.scale_log2 = scale * pkv::kLog2e;
  return cuda_status(pkv::launch_prefill_bf16(p, st));
}

int paged_kv_append(const void* k_new, const void* v_new, const int32_t* cu_new,
                    const int32_t* start_pos, const int32_t* block_table, int max_pages_per_seq,
                    int num_seqs, int num_new, void* k_pages, void* v_pages, int num_pages,
                    int page_size, int H_kv, int d, int dtype, void* stream) {
  if (num_new < 0 || num_seqs < 1 || max_pages_per_seq < 1 || num_pages < 1 || H_kv < 1 ||
      !pow2(page_size) || page_size < 16 || page_size > 256 ||
      (dtype != PKV_BF16 && dtype != PKV_F32))
    return PKV_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return PKV_ERR_UNSUPPORTED;
  if (num_new == 0) return PKV_OK;
  if (!aligned16(k_new) || !aligned16(v_new) || !aligned16(k_pages) || !aligned16(v_pages) ||
      !aligned4(cu_new) || !aligned4(start_pos) || !aligned4(block_table))
    return PKV_ERR_INVALID_ARG;
  if ((long long)num_pages * page_size > (1LL << 31)) return PKV_ERR_UNSUPPORTED;
  unsigned int* err = nullptr;
  if (int r = error_word(&err)) return r;
  pkv::AppendParams p{};
  p.k_new = k_new, p.v_new = v_new, p.cu_new = cu_new, p.start_pos = start_pos;
  p.block_table = block_table, p.k_pages = k_pages, p.v_pages = v_pages, p.err = err;
  p.num_seqs = num_seqs, p.num_new = num_new, p.max_pages = max_pages_per_seq;
  p.num_pages = num_pages, p.page_size = page_size, p.page_shift = log2i(page_size);
  p.row_bytes = (size_t)H_kv * d * (dtype == PKV_BF16 ? 2 : 4);
  return cuda_status(pkv::launch_append(p, static_cast<cudaStream_t>(stream)));
}

int paged_kv_copy_pages(void* k_pages, void* v_pages, const int32_t* src, const int32_t* dst,
                        int n, int num_pages, int page_size, int H_kv, int d, int dtype,
                        void* stream) {
  if (n < 0 || num_pages < 1 || H_kv < 1 || !pow2(page_size) || page_size < 16 ||
      page_size > 256 || (dtype != PKV_BF16 && dtype != PKV_F32))
    return PKV_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return PKV_ERR_UNSUPPORTED;
  if (n == 0) return PKV_OK;
  if (!aligned16(k_pages) || !aligned16(v_pages) || !aligned4(src) || !aligned4(dst))
    return PKV_ERR_INVALID_ARG;
  unsigned int* err = nullptr;
  if (int r = error_word(&err)) return r;
  pkv::CopyPagesParams p{};
  p.k_pages = k_pages, p.v_pages = v_pages, p.src = src, p.dst = dst, p.err = err;
  p.n = n, p.num_pages = num_pages;
  p.page_bytes = (size_t)page_size * H_kv * d * (dtype == PKV_BF16 ? 2 : 4);
  return cuda_status(pkv::launch_copy_pages(p, static_cast<cudaStream_t>(stream)));
}

int pkv_last_device_error(void* stream, unsigned int* bits) {
  unsigned int* err = nullptr;
  if (int r = error_word(&err)) return r;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return PKV_ERR_CUDA;
  unsigned int v = 0;
  if (cudaMemcpy(&v, err, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) return PKV_ERR_CUDA;
  const unsigned int zero = 0;
  if (cudaMemcpy(err, &zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess)
    return PKV_ERR_CUDA;
  if (bits) *bits = v;
  if (v & PKV_DEVERR_TIMEOUT) return PKV_ERR_TIMEOUT;
  if (v & (PKV_DEVERR_BAD_PAGE | PKV_DEVERR_BAD_LEN)) return PKV_ERR_BAD_TABLE;
  return PKV_OK;
}

}  // extern "C"
