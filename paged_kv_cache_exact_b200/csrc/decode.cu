// Paged decode (one query token per sequence), bf16, head dim 128.
//
// "What is Paged FlashAttention?", section "How does it work?": locate each
// token's page through the block table, load K/V straight from the page,
// compute scores and keep a numerically stable running softmax, accumulate
// the output, never gathering the cache into a contiguous copy.  Its section
// "Does it change the attention result or complexity?" notes that decode is
// bound by reading the cache, so this kernel is organised around HBM reads:
//
// * grid = (split, head, sequence).  Each CTA owns `split_tokens` consecutive
//   keys of one (sequence, head) so that long and short sequences spread over
//   many equal-sized CTAs.
// * The split's block-table entries are staged in shared memory once, so the
//   K/V loads in the main loop never wait on a dependent table load.
// * A half-warp owns one token row at a time: 16 lanes x 16-byte vector loads
//   cover the 256-byte row of K (and of V) for one head; the q.k dot product is
//   reduced with four xor-shuffles inside the half-warp.
// * Each half-warp keeps its own running (max, sum, O); the 8 half-warps are
//   merged in shared memory, and the splits of a sequence are merged by
//   `combine_kernel` with the same log-sum-exp algebra (scores are kept in
//   base-2 units: q is pre-multiplied by scale * log2(e)).
#include "common.cuh"

namespace pkv {
namespace {

constexpr int D = 128;
constexpr int kThreads = 128;           // 4 warps = 8 half-warps
constexpr int kHalfWarps = kThreads / 16;
constexpr int kMaxSplitPages = 256;     // table entries staged per CTA
constexpr int kMaxSplits = 1024;        // splits merged per (sequence, head)

template <int U>
__global__ void __launch_bounds__(kThreads)
decode_split_kernel(const DecodeParams p) {
  const int split = blockIdx.x, h = blockIdx.y, s = blockIdx.z;
  const int tid = threadIdx.x;

  int L = p.seq_lens[s];
  const int cap = min(p.max_seq_len, p.max_pages * p.page_size);
  if (L < 1 || L > cap) {
    if (split == 0 && h == 0 && tid == 0) flag_error(p.err, PKV_DEVERR_BAD_LEN);
    L = max(0, min(L, cap));
  }
  const size_t sh = (size_t)s * p.H + h;
  if (L <= 0) {                                   // invalid length: defined output (zeros)
    if (split == 0) p.out[sh * D + tid] = __float2bfloat16_rn(0.f);
    return;
  }
  const int t_begin = split * p.split_tokens;
  if (t_begin >= L) return;
  const int t_end = min(L, t_begin + p.split_tokens);
  const int nsplit = (L + p.split_tokens - 1) / p.split_tokens;
  const int kvh = h / (p.H / p.H_kv);

  __shared__ int s_pages[kMaxSplitPages];
  __shared__ float s_m[kHalfWarps], s_l[kHalfWarps];
  __shared__ float s_acc[kHalfWarps][D];

  // Stage this split's page ids (bad ids become -1: skipped and flagged).
  const int lp0 = t_begin >> p.page_shift;
  const int lp1 = (t_end - 1) >> p.page_shift;
  for (int i = tid; i <= lp1 - lp0; i += kThreads) {
    int phys = p.block_table[(size_t)s * p.max_pages + lp0 + i];
    if (phys < 0 || phys >= p.num_pages) {
      flag_error(p.err, PKV_DEVERR_BAD_PAGE);
      phys = -1;
    }
    s_pages[i] = phys;
  }

  const int hl = tid & 15;           // lane in half-warp: dims [8*hl, 8*hl + 8)
  const int hw = tid >> 4;           // half-warp id
  float qf[8];
  {
    const uint4 qv = *reinterpret_cast<const uint4*>(p.q + ((size_t)s * p.H + h) * D + hl * 8);
    const uint32_t w[4] = {qv.x, qv.y, qv.z, qv.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      qf[2 * i] = bf16lo(w[i]) * p.scale_log2;
      qf[2 * i + 1] = bf16hi(w[i]) * p.scale_log2;
    }
  }
  __syncthreads();

  const size_t row_stride = (size_t)p.H_kv * D;    // elements between tokens of a page
  const __nv_bfloat16* kbase = p.k_pages + (size_t)kvh * D + hl * 8;
  const __nv_bfloat16* vbase = p.v_pages + (size_t)kvh * D + hl * 8;
  const int pmask = p.page_size - 1;

  float m = -INFINITY, l = 0.f;
  float acc[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] = 0.f;

  // The loop bound is uniform per warp (both half-warps take the same trip
  // count), so the full-warp shuffles below are always converged.
  for (int tb = t_begin + (hw >> 1) * 2 * U; tb < t_end; tb += kHalfWarps * U) {
    const int t0 = tb + (hw & 1) * U;
    uint4 kv[U], vv[U];
    bool ok[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int t = t0 + u;
      int phys = -1;
      if (t < t_end) phys = s_pages[(t >> p.page_shift) - lp0];
      ok[u] = phys >= 0;
      const size_t row = ((size_t)phys << p.page_shift) + (t & pmask);
      if (ok[u]) {
        kv[u] = ldg_nc_v4(kbase + row * row_stride);
        vv[u] = ldg_nc_v4(vbase + row * row_stride);
      } else {
        kv[u] = make_uint4(0, 0, 0, 0);
        vv[u] = make_uint4(0, 0, 0, 0);
      }
    }
    float sc[U];
    float mx = -INFINITY;
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const uint32_t w[4] = {kv[u].x, kv[u].y, kv[u].z, kv[u].w};
      float dot = 0.f;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        dot = fmaf(qf[2 * i], bf16lo(w[i]), dot);
        dot = fmaf(qf[2 * i + 1], bf16hi(w[i]), dot);
      }
      dot += __shfl_xor_sync(0xffffffffu, dot, 8);
      dot += __shfl_xor_sync(0xffffffffu, dot, 4);
      dot += __shfl_xor_sync(0xffffffffu, dot, 2);
      dot += __shfl_xor_sync(0xffffffffu, dot, 1);
      sc[u] = ok[u] ? dot : -INFINITY;
      mx = fmaxf(mx, sc[u]);
    }
    const float m_new = fmaxf(m, mx);
    if (m_new == -INFINITY) continue;                 // nothing visible yet
    const float alpha = ex2(m - m_new);               // m = -inf -> 0
    l *= alpha;
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] *= alpha;
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const float pr = ex2(sc[u] - m_new);            // masked -> 0
      l += pr;
      const uint32_t w[4] = {vv[u].x, vv[u].y, vv[u].z, vv[u].w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        acc[2 * i] = fmaf(pr, bf16lo(w[i]), acc[2 * i]);
        acc[2 * i + 1] = fmaf(pr, bf16hi(w[i]), acc[2 * i + 1]);
      }
    }
    m = m_new;
  }

  // Merge the half-warps of this CTA.
  if (hl == 0) {
    s_m[hw] = m;
    s_l[hw] = l;
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) s_acc[hw][hl * 8 + i] = acc[i];
  __syncthreads();

  float M = -INFINITY;
#pragma unroll
  for (int j = 0; j < kHalfWarps; ++j) M = fmaxf(M, s_m[j]);
  float o = 0.f, lsum = 0.f;
  if (M != -INFINITY) {
#pragma unroll
    for (int j = 0; j < kHalfWarps; ++j) {
      const float w = ex2(s_m[j] - M);
      o = fmaf(w, s_acc[j][tid], o);
      lsum = fmaf(w, s_l[j], lsum);
    }
  }
  if (nsplit == 1) {
    p.out[sh * D + tid] = __float2bfloat16_rn(lsum > 0.f ? o / lsum : 0.f);
  } else {
    p.ws_o[(sh * p.max_splits + split) * D + tid] = o;
    if (tid == 0) p.ws_ml[sh * p.max_splits + split] = make_float2(M, lsum);
  }
}

// Log-sum-exp merge of the splits of one (sequence, head).
__global__ void __launch_bounds__(D) combine_kernel(const DecodeParams p) {
  const int h = blockIdx.x, s = blockIdx.y, tid = threadIdx.x;
  int L = p.seq_lens[s];
  const int cap = min(p.max_seq_len, p.max_pages * p.page_size);
  L = max(0, min(L, cap));
  const int nsplit = (L + p.split_tokens - 1) / p.split_tokens;
  if (nsplit <= 1) return;                          // written by the split kernel
  const size_t sh = (size_t)s * p.H + h;
  const float2* ml = p.ws_ml + sh * p.max_splits;
  __shared__ float s_w[kMaxSplits];
  __shared__ float s_red[D / 32];
  __shared__ float s_M, s_L;
  // max over splits
  float M = -INFINITY;
  for (int j = tid; j < nsplit; j += D) M = fmaxf(M, ml[j].x);
#pragma unroll
  for (int o = 16; o; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  if ((tid & 31) == 0) s_red[tid >> 5] = M;
  __syncthreads();
  if (tid == 0) {
    float mm = s_red[0];
    for (int i = 1; i < D / 32; ++i) mm = fmaxf(mm, s_red[i]);
    s_M = mm;
  }
  __syncthreads();
  M = s_M;
  float lsum = 0.f;
  for (int j = tid; j < nsplit; j += D) {
    const float2 v = ml[j];
    const float w = (M == -INFINITY) ? 0.f : ex2(v.x - M);
    s_w[j] = w;
    lsum = fmaf(w, v.y, lsum);
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) lsum += __shfl_xor_sync(0xffffffffu, lsum, o);
  __syncthreads();
  if ((tid & 31) == 0) s_red[tid >> 5] = lsum;
  __syncthreads();
  if (tid == 0) {
    float t = 0.f;
    for (int i = 0; i < D / 32; ++i) t += s_red[i];
    s_L = t;
  }
  __syncthreads();
  const float* po = p.ws_o + sh * p.max_splits * D + tid;
  float o = 0.f;
  for (int j = 0; j < nsplit; ++j) o = fmaf(s_w[j], po[(size_t)j * D], o);
  p.out[sh * D + tid] = __float2bfloat16_rn(s_L > 0.f ? o / s_L : 0.f);
}

}  // namespace

void decode_plan(int num_seqs, int H, int max_seq_len, int page_size,
                 int* split_tokens, int* max_splits) {
  // Fixed-size splits: enough CTAs to fill the GPU several times over, each
  // long enough to amortise its merge.  A power of two >= the page size, so a
  // split never shares a page with the next one unless pages are larger.
  int st = 256;
  const long long work = (long long)num_seqs * H;
  // few (sequence, head) pairs: shorter splits for more parallelism
  while (st > 64 && work * ((max_seq_len + st - 1) / st) < 148LL * 16) st >>= 1;
  if (st < page_size) st = page_size;             // a split holds whole pages
  // very long sequences: cap the number of splits (workspace, combine cost)
  while ((max_seq_len + st - 1) / st > kMaxSplits) st <<= 1;
  *split_tokens = st;
  *max_splits = (max_seq_len + st - 1) / st;
}

cudaError_t launch_decode_bf16(const DecodeParams& p, cudaStream_t stream) {
  dim3 grid(p.max_splits, p.H, p.num_seqs);
  decode_split_kernel<4><<<grid, kThreads, 0, stream>>>(p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (p.max_splits > 1) {
    combine_kernel<<<dim3(p.H, p.num_seqs), D, 0, stream>>>(p);
    e = cudaGetLastError();
  }
  return e;
}

}  // namespace pkv
