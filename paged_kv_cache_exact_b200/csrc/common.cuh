// Shared device helpers and the internal launcher interface (not part of the C ABI).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "../../include/pkv.h"

#define PKV_DEVINLINE __device__ __forceinline__

namespace pkv {

constexpr float kLog2e = 1.4426950408889634f;

// Hardware base-2 exponential (MUFU ex2; flushes denormal results to zero).
// exp2(-inf) = +0, which masked scores rely on.
PKV_DEVINLINE float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Two floats -> packed bf16x2 (round to nearest even); `lo` in bits 0..15.
PKV_DEVINLINE uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

PKV_DEVINLINE float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
PKV_DEVINLINE float bf16hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

PKV_DEVINLINE uint4 ldg_nc_v4(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
  return r;
}

PKV_DEVINLINE void flag_error(unsigned int* err, unsigned int bits) {
  if (err) atomicOr(err, bits);
}

// ----------------------------------------------------------------------------
// Launchers, one per kernel family.  Arguments are validated by the C ABI layer
// before any of these is called.
// ----------------------------------------------------------------------------

struct DecodeParams {
  const __nv_bfloat16* q;        // [S, H, 1, d]
  const __nv_bfloat16* k_pages;  // [P, ps, H_kv, d]
  const __nv_bfloat16* v_pages;
  const int32_t* block_table;    // [S, max_pages]
  const int32_t* seq_lens;       // [S]
  __nv_bfloat16* out;            // [S, H, 1, d]
  float* ws_o;                   // [S, H, max_splits, d]   (unnormalised partial O)
  float2* ws_ml;                 // [S, H, max_splits]      (max in log2 units, sum)
  unsigned int* err;
  int num_seqs, H, H_kv, page_size, page_shift, num_pages, max_pages, max_seq_len;
  int split_tokens, max_splits;
  float scale_log2;              // scale * log2(e)
};

struct SimtParams {
  const float* q;        // [B, H, q_len, d]
  const float* k;        // contiguous: [B, H_kv, kv_len, d]; paged: [P, ps, H_kv, d]
  const float* v;
  const int32_t* block_table;  // paged only
  const int32_t* seq_lens;     // paged only
  float* out;            // [B, H, q_len, d]
  unsigned int* err;
  int B, H, H_kv, q_len, kv_len, d;     // kv_len: contiguous only
  int paged, page_size, page_shift, num_pages, max_pages, max_seq_len;
  int causal;
  float scale_log2;
};

struct PrefillParams {
  const void* Q;  // [B, H, q_len, d] bf16
  const void* K;  // contiguous: [B, H_kv, kv_len, d]; paged: [P, ps, H_kv, d]
  const void* V;
  void* O;        // [B, H, q_len, d] bf16
  const int32_t* block_table;
  const int32_t* seq_lens;
  unsigned int* err;
  int B, H, H_kv, q_len, kv_len, d;
  int paged, page_size, page_shift, num_pages, max_pages, max_seq_len;
  int causal;
  float scale_log2;
  int head_group;   // (batch, head) pairs scheduled together (set by the launcher)
  int fp8_qk;       // Q and K are e4m3 (contiguous only); V and O stay bf16
  // Failure-path controls; zero (the value-initialised default) means off.
  // wait_limit_ns bounds every pipeline wait (0 = the default of 2 s).
  // stall_tile_plus1 = j + 1 is a test hook only: the loader of each CTA's
  // first work item skips the K load of K/V tile j, so the MMA issuer's wait
  // for it runs out; the public entry points leave it 0.
  unsigned long long wait_limit_ns;
  int stall_tile_plus1;
};

struct AppendParams {
  const void* k_new;           // [num_new, H_kv, d]
  const void* v_new;
  const int32_t* cu_new;       // [num_seqs + 1]
  const int32_t* start_pos;    // [num_seqs]
  const int32_t* block_table;  // [num_seqs, max_pages]
  void* k_pages;               // [P, ps, H_kv, d]
  void* v_pages;
  unsigned int* err;
  int num_seqs, num_new, max_pages, num_pages, page_size, page_shift;
  size_t row_bytes;            // H_kv * d * element size
};

struct CopyPagesParams {
  void* k_pages;
  void* v_pages;
  const int32_t* src;
  const int32_t* dst;
  unsigned int* err;
  int n, num_pages;
  size_t page_bytes;           // page_size * H_kv * d * element size
};

// Split plan for decode: fixed-size key chunks per (sequence, head).
void decode_plan(int num_seqs, int H, int max_seq_len, int page_size,
                 int* split_tokens, int* max_splits);

cudaError_t launch_decode_bf16(const DecodeParams& p, cudaStream_t stream);
cudaError_t launch_simt_f32(const SimtParams& p, cudaStream_t stream);
cudaError_t launch_prefill_bf16(const PrefillParams& p, cudaStream_t stream);
cudaError_t launch_append(const AppendParams& p, cudaStream_t stream);
cudaError_t launch_copy_pages(const CopyPagesParams& p, cudaStream_t stream);

// Device address of the library's error word on the current device.
int device_error_word(unsigned int** out);

// pkv_status of a launcher's result: cudaErrorNotSupported (a configuration
// with no kernel) -> PKV_ERR_UNSUPPORTED, any other failure -> PKV_ERR_CUDA.
int cuda_status(cudaError_t e);

}  // namespace pkv
