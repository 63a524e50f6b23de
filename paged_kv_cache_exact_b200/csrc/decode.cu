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
#include <mutex>

#include "common.cuh"

namespace pkv {
namespace {
PKV_DEVINLINE uint32_t sm100_smem_addr(const void* ptr) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(ptr));
}
}  // namespace
}  // namespace pkv

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

// Log-sum-exp merge of the splits of one (sequence, head), for the per-head
// plan: up to kMaxSplits splits per pair, a 128-thread CTA each (one thread
// per head dim) so that many partial loads are in flight.
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


// The same merge for the grouped-query plan (a few long splits per head),
// one warp per (sequence, head):
// lane i owns head dims 4i .. 4i+3 (one 16-byte load per split).  Launched as
// a programmatic dependent of the split kernel: the grid may be scheduled
// while the split kernel drains, and waits here until all of its partials are
// written and visible.
constexpr int kCombineWarps = 8;
__global__ void __launch_bounds__(kCombineWarps * 32) combine_warp_kernel(const DecodeParams p) {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const long long sh = (long long)blockIdx.x * kCombineWarps + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (sh >= (long long)p.num_seqs * p.H) return;
  int L = p.seq_lens[sh / p.H];
  const int cap = min(p.max_seq_len, p.max_pages * p.page_size);
  L = max(0, min(L, cap));
  const int nsplit = (L + p.split_tokens - 1) / p.split_tokens;
  if (nsplit <= 1) return;                          // written by the split kernel
  const float2* ml = p.ws_ml + sh * p.max_splits;
  float M = -INFINITY;
  for (int j = lane; j < nsplit; j += 32) M = fmaxf(M, ml[j].x);
#pragma unroll
  for (int o = 16; o; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  float lsum = 0.f;
  for (int j = lane; j < nsplit; j += 32) {
    const float2 v = ml[j];
    lsum = fmaf(M == -INFINITY ? 0.f : ex2(v.x - M), v.y, lsum);
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) lsum += __shfl_xor_sync(0xffffffffu, lsum, o);
  const float4* po = reinterpret_cast<const float4*>(p.ws_o + sh * p.max_splits * D) + lane;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int j = 0; j < nsplit; ++j) {
    const float w = M == -INFINITY ? 0.f : ex2(ml[j].x - M);
    const float4 x = po[(size_t)j * (D / 4)];
    acc.x = fmaf(w, x.x, acc.x);
    acc.y = fmaf(w, x.y, acc.y);
    acc.z = fmaf(w, x.z, acc.z);
    acc.w = fmaf(w, x.w, acc.w);
  }
  const bool pos = lsum > 0.f;
  __nv_bfloat162* out = reinterpret_cast<__nv_bfloat162*>(p.out + sh * D) + 2 * lane;
  out[0] = __floats2bfloat162_rn(pos ? acc.x / lsum : 0.f, pos ? acc.y / lsum : 0.f);
  out[1] = __floats2bfloat162_rn(pos ? acc.z / lsum : 0.f, pos ? acc.w / lsum : 0.f);
}


// ---------------------------------------------------------------------------
// Grouped-query decode (H > H_kv): one CTA per (split, kv head, sequence,
// group of up to 16 query heads).  Every K/V row of the split is read from
// HBM once, into shared memory, and serves all query heads that share the kv
// head ("Flash Attention: Fast, Memory-Efficient Attention for LLMs", section
// "Attention Variants: MHA, GQA, MQA").  With 2..16 query rows per kv head the
// scores and the PV product are small matrix products, done on the tensor
// cores with mma.sync m16n8k16 (bf16 in, f32 accumulate): M = 16 query heads
// (padded), N = 8 tokens (QK^T) or 8 head dims (PV), K = 16.  Each of the 4
// warps streams its own 16-token chunks through a 2-stage cp.async ring
// (XOR-swizzled rows, so ldmatrix reads are conflict-free), keeps a running
// (max, sum, O) per query head, and the warps and splits are merged with the
// same log-sum-exp algebra as the per-head kernel.
// ---------------------------------------------------------------------------
constexpr int kGqaWarps = 4;
constexpr int kGqaThreads = kGqaWarps * 32;
constexpr int kChunk = 16;                          // tokens per warp step
constexpr int kRowBytes = D * 2;                    // 256 B per token row
constexpr int kStageBytes = kChunk * kRowBytes;     // 4 KB per matrix per stage
// Ring depth per warp and the split-planning target: 2 stages keep shared
// memory at 65 KB per CTA (3 CTAs = 12 warps per SM), which measured faster
// than 3 stages at 2 CTAs per SM; finer splits (more CTAs per SM) measured
// slower.
constexpr int kGqaStages = 2;                        // cp.async ring depth per warp
constexpr int kGqaCtasPerSm = 8;                     // split planning target
constexpr int kWarpSmem = kGqaStages * 2 * kStageBytes;   // stages x (K, V)

PKV_DEVINLINE void cp_async16(uint32_t dst, const void* src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
               "r"(valid ? 16 : 0)
               : "memory");
}
PKV_DEVINLINE void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
PKV_DEVINLINE void cp_async_wait_1() { asm volatile("cp.async.wait_group 1;" ::: "memory"); }
PKV_DEVINLINE void cp_async_wait_0() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

PKV_DEVINLINE void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
PKV_DEVINLINE void ldsm_x4_t(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
// d[16x8 f32] += a[16x16 bf16, row-major] * b[16x8 bf16, col-major]
PKV_DEVINLINE void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                  uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// byte offset of 16-byte chunk c of token row r inside a stage (rows of 256 B)
PKV_DEVINLINE uint32_t swz(int r, int c) { return r * kRowBytes + ((c ^ (r & 7)) << 4); }

__global__ void __launch_bounds__(kGqaThreads)
decode_gqa_kernel(const DecodeParams p) {
  extern __shared__ __align__(128) uint8_t gsm[];
  asm volatile("griddepcontrol.launch_dependents;");   // the combine may be scheduled
  const int split = blockIdx.x, s = blockIdx.z;
  const int group = p.H / p.H_kv;                    // query heads per kv head
  const int n_hg = (group + 15) / 16;                // 16-head groups per kv head
  const int kvh = blockIdx.y / n_hg;
  const int h0 = kvh * group + (blockIdx.y % n_hg) * 16;   // first query head of this CTA
  const int nh = min(16, kvh * group + group - h0);        // query heads in this CTA
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, t4 = lane & 3;

  int L = p.seq_lens[s];
  const int cap = min(p.max_seq_len, p.max_pages * p.page_size);
  if (L < 1 || L > cap) {
    if (split == 0 && blockIdx.y == 0 && tid == 0) flag_error(p.err, PKV_DEVERR_BAD_LEN);
    L = max(0, min(L, cap));
  }
  if (L <= 0) {
    if (split == 0)
      for (int i = tid; i < nh * D; i += kGqaThreads)
        p.out[((size_t)s * p.H + h0 + i / D) * D + i % D] = __float2bfloat16_rn(0.f);
    return;
  }
  const int t_begin = split * p.split_tokens;
  if (t_begin >= L) return;
  const int t_end = min(L, t_begin + p.split_tokens);
  const int nsplit = (L + p.split_tokens - 1) / p.split_tokens;

  // shared memory: per-warp K/V rings, then the split's page ids
  int* s_pages = reinterpret_cast<int*>(gsm + kGqaWarps * kWarpSmem);
  const int lp0 = t_begin >> p.page_shift;
  const int lp1 = (t_end - 1) >> p.page_shift;
  for (int i = tid; i <= lp1 - lp0; i += kGqaThreads) {
    int phys = p.block_table[(size_t)s * p.max_pages + lp0 + i];
    if (phys < 0 || phys >= p.num_pages) {
      flag_error(p.err, PKV_DEVERR_BAD_PAGE);
      phys = -1;
    }
    s_pages[i] = phys;
  }

  // Q as the A operand (rows = query heads, padded to 16; k = head dim),
  // pre-rounded bf16 exactly as stored.
  uint32_t qa[D / 16][4];
  {
    const __nv_bfloat16* qs = p.q + ((size_t)s * p.H + h0) * D;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      const int c0 = 16 * kk + 2 * t4;
      const uint32_t* r0 = reinterpret_cast<const uint32_t*>(qs + (size_t)g * D);
      const uint32_t* r1 = reinterpret_cast<const uint32_t*>(qs + (size_t)(g + 8) * D);
      qa[kk][0] = g < nh ? r0[c0 / 2] : 0u;
      qa[kk][1] = g + 8 < nh ? r1[c0 / 2] : 0u;
      qa[kk][2] = g < nh ? r0[(c0 + 8) / 2] : 0u;
      qa[kk][3] = g + 8 < nh ? r1[(c0 + 8) / 2] : 0u;
    }
  }
  __syncthreads();                                   // s_pages ready

  const uint32_t wbase = sm100_smem_addr(gsm) + warp * kWarpSmem;
  auto k_stage = [&](int stage) { return wbase + stage * 2 * kStageBytes; };
  auto v_stage = [&](int stage) { return wbase + stage * 2 * kStageBytes + kStageBytes; };
  const size_t row_stride = (size_t)p.H_kv * D;
  const __nv_bfloat16* kbase = p.k_pages + (size_t)kvh * D;
  const __nv_bfloat16* vbase = p.v_pages + (size_t)kvh * D;
  const int pmask = p.page_size - 1;

  // this lane's copies: token rows (lane / 16) + 2 i, 16-byte column chunk lane % 16
  auto prefetch = [&](int chunk, int stage) {
    const int cc = lane & 15;
#pragma unroll
    for (int i = 0; i < kChunk / 2; ++i) {
      const int r = (lane >> 4) + 2 * i;
      const int tok = t_begin + chunk * kChunk + r;
      int phys = -1;
      if (tok < t_end) phys = s_pages[(tok >> p.page_shift) - lp0];
      const bool ok = phys >= 0;
      const size_t row = ok ? (((size_t)phys << p.page_shift) + (tok & pmask)) : 0;
      cp_async16(k_stage(stage) + swz(r, cc), kbase + row * row_stride + cc * 8, ok);
      cp_async16(v_stage(stage) + swz(r, cc), vbase + row * row_stride + cc * 8, ok);
    }
  };

  float o[D / 8][4];
#pragma unroll
  for (int i = 0; i < D / 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
  float m_lo = -INFINITY, m_hi = -INFINITY, l_lo = 0.f, l_hi = 0.f;   // rows g, g + 8

  const int n_chunks = (t_end - t_begin + kChunk - 1) / kChunk;
  // ring of kGqaStages chunks per warp: this warp's chunks are warp, warp + 4, ...
#pragma unroll
  for (int i = 0; i < kGqaStages - 1; ++i) {
    if (warp + i * kGqaWarps < n_chunks) prefetch(warp + i * kGqaWarps, i);
    cp_async_commit();
  }
  int st = 0;
  for (int c = warp; c < n_chunks; c += kGqaWarps) {
    const int ahead = c + (kGqaStages - 1) * kGqaWarps;
    if (ahead < n_chunks) prefetch(ahead, (st + kGqaStages - 1) % kGqaStages);
    cp_async_commit();
    cp_async_wait_1();                               // this chunk's group is complete
    __syncwarp();

    // S = Q K^T for 16 tokens: two n-tiles of 8 tokens, each accumulated in
    // two halves of the head dimension (two independent MMA chains)
    float sc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
    float sd[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      const int mi = lane >> 3, ri = lane & 7;
      uint32_t b[4];
      ldsm_x4(k_stage(st) + swz(8 * (mi >> 1) + ri, 2 * kk + (mi & 1)), b);
      mma_bf16_16816(kk & 1 ? sd[0] : sc[0], qa[kk], b[0], b[1]);
      mma_bf16_16816(kk & 1 ? sd[1] : sc[1], qa[kk], b[2], b[3]);
    }
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) sc[nt][e] += sd[nt][e];
    // online softmax per query head (rows g and g + 8), base 2.  A chunk lies
    // in one page (pages hold >= 16 tokens, chunks start 16-aligned); keys of
    // a page outside the pool are left out.
    const int tok0 = t_begin + c * kChunk;
    const bool page_ok = s_pages[(tok0 >> p.page_shift) - lp0] >= 0;
    float mx_lo = -INFINITY, mx_hi = -INFINITY;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const bool valid = page_ok && tok0 + 8 * nt + 2 * t4 + e < t_end;
        sc[nt][e] = valid ? sc[nt][e] * p.scale_log2 : -INFINITY;
        sc[nt][2 + e] = valid ? sc[nt][2 + e] * p.scale_log2 : -INFINITY;
        mx_lo = fmaxf(mx_lo, sc[nt][e]);
        mx_hi = fmaxf(mx_hi, sc[nt][2 + e]);
      }
    mx_lo = fmaxf(mx_lo, __shfl_xor_sync(0xffffffffu, mx_lo, 1));
    mx_lo = fmaxf(mx_lo, __shfl_xor_sync(0xffffffffu, mx_lo, 2));
    mx_hi = fmaxf(mx_hi, __shfl_xor_sync(0xffffffffu, mx_hi, 1));
    mx_hi = fmaxf(mx_hi, __shfl_xor_sync(0xffffffffu, mx_hi, 2));
    // Reference max per query head, moved only when the chunk's max exceeds
    // it by more than 2^8 (exact: O and l share it; p stays <= 2^8).
    const float mn_lo = mx_lo > m_lo + 8.f || (m_lo == -INFINITY && mx_lo != -INFINITY) ? mx_lo : m_lo;
    const float mn_hi = mx_hi > m_hi + 8.f || (m_hi == -INFINITY && mx_hi != -INFINITY) ? mx_hi : m_hi;
    // rescale factors: 1 when the reference stays (also -inf, no key yet), 0 from -inf
    const float a_lo = mn_lo == m_lo ? 1.f : ex2(m_lo - mn_lo);
    const float a_hi = mn_hi == m_hi ? 1.f : ex2(m_hi - mn_hi);
    const float sub_lo = mn_lo == -INFINITY ? 0.f : mn_lo;
    const float sub_hi = mn_hi == -INFINITY ? 0.f : mn_hi;
    const bool moved = __any_sync(0xffffffffu, mn_lo != m_lo || mn_hi != m_hi);
    m_lo = mn_lo;
    m_hi = mn_hi;
    float pr[2][4];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        pr[nt][e] = ex2(sc[nt][e] - sub_lo);
        pr[nt][2 + e] = ex2(sc[nt][2 + e] - sub_hi);
      }
    l_lo = l_lo * a_lo + (pr[0][0] + pr[0][1]) + (pr[1][0] + pr[1][1]);
    l_hi = l_hi * a_hi + (pr[0][2] + pr[0][3]) + (pr[1][2] + pr[1][3]);
    if (moved) {                                     // warp-uniform
#pragma unroll
      for (int i = 0; i < D / 8; ++i) {
        o[i][0] *= a_lo;
        o[i][1] *= a_lo;
        o[i][2] *= a_hi;
        o[i][3] *= a_hi;
      }
    }
    // P as the A operand: k = the chunk's 16 tokens
    uint32_t pa[4];
    pa[0] = pack_bf16x2(pr[0][0], pr[0][1]);
    pa[1] = pack_bf16x2(pr[0][2], pr[0][3]);
    pa[2] = pack_bf16x2(pr[1][0], pr[1][1]);
    pa[3] = pack_bf16x2(pr[1][2], pr[1][3]);
    // O += P V: 16 n-tiles of 8 head dims
#pragma unroll
    for (int nd = 0; nd < D / 8; nd += 2) {
      const int mi = lane >> 3, ri = lane & 7;
      uint32_t b[4];
      ldsm_x4_t(v_stage(st) + swz(8 * (mi & 1) + ri, nd + (mi >> 1)), b);
      mma_bf16_16816(o[nd], pa, b[0], b[1]);
      mma_bf16_16816(o[nd + 1], pa, b[2], b[3]);
    }
    __syncwarp();                                    // stage st may be refilled
    st = (st + 1) % kGqaStages;
  }
  cp_async_wait_0();
  l_lo += __shfl_xor_sync(0xffffffffu, l_lo, 1);
  l_lo += __shfl_xor_sync(0xffffffffu, l_lo, 2);
  l_hi += __shfl_xor_sync(0xffffffffu, l_hi, 1);
  l_hi += __shfl_xor_sync(0xffffffffu, l_hi, 2);
  __syncthreads();                                   // rings no longer read: reuse as merge buffers

  // merge the warps: per warp, O [16][D] f32 and (m, l) [16]
  float* s_o = reinterpret_cast<float*>(gsm);                       // [warps][16][D]
  float* s_ml = s_o + kGqaWarps * 16 * D;                           // [warps][16][2]
#pragma unroll
  for (int nd = 0; nd < D / 8; ++nd) {
    const int col = 8 * nd + 2 * t4;
    s_o[(warp * 16 + g) * D + col] = o[nd][0];
    s_o[(warp * 16 + g) * D + col + 1] = o[nd][1];
    s_o[(warp * 16 + g + 8) * D + col] = o[nd][2];
    s_o[(warp * 16 + g + 8) * D + col + 1] = o[nd][3];
  }
  if (t4 == 0) {
    s_ml[(warp * 16 + g) * 2] = m_lo;
    s_ml[(warp * 16 + g) * 2 + 1] = l_lo;
    s_ml[(warp * 16 + g + 8) * 2] = m_hi;
    s_ml[(warp * 16 + g + 8) * 2 + 1] = l_hi;
  }
  __syncthreads();
  for (int i = tid; i < nh * D; i += kGqaThreads) {
    const int r = i / D, col = i % D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kGqaWarps; ++w) M = fmaxf(M, s_ml[(w * 16 + r) * 2]);
    float acc = 0.f, lsum = 0.f;
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < kGqaWarps; ++w) {
        const float wt = ex2(s_ml[(w * 16 + r) * 2] - M);
        acc = fmaf(wt, s_o[(w * 16 + r) * D + col], acc);
        lsum = fmaf(wt, s_ml[(w * 16 + r) * 2 + 1], lsum);
      }
    }
    const size_t sh = (size_t)s * p.H + h0 + r;
    if (nsplit == 1) {
      p.out[sh * D + col] = __float2bfloat16_rn(lsum > 0.f ? acc / lsum : 0.f);
    } else {
      p.ws_o[(sh * p.max_splits + split) * D + col] = acc;
      if (col == 0) p.ws_ml[sh * p.max_splits + split] = make_float2(M, lsum);
    }
  }
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

// The grouped-query merge as a programmatic dependent launch of the split
// kernel just enqueued on `stream` (it waits for that kernel's results
// itself).  Measured against a plain launch of the CTA merge: 201.9 against
// 204.5 us on 64 sequences x 64 query heads over 8 kv heads; on the per-head
// plan (32 splits per pair) the CTA merge with a plain launch stays ahead.
static cudaError_t launch_combine(const DecodeParams& q, cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(((long long)q.num_seqs * q.H + kCombineWarps - 1) / kCombineWarps));
  cfg.blockDim = dim3(kCombineWarps * 32);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, combine_warp_kernel, q);
}

cudaError_t launch_decode_bf16(const DecodeParams& p, cudaStream_t stream) {
  cudaError_t e;
  if (p.H > p.H_kv) {
    // grouped heads: one CTA per (split, kv head, 16 query heads, sequence)
    const int n_hg = (p.H / p.H_kv + 15) / 16;
    const size_t smem = kGqaWarps * kWarpSmem + kMaxSplitPages * sizeof(int);
    // The attribute is per device; callers on several host threads may get
    // here at once, so the once-per-device record is kept under a lock.
    static bool attr_set[64] = {};
    static std::mutex attr_mu;
    int dev = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    {
      std::lock_guard<std::mutex> lock(attr_mu);
      if (dev < 0 || dev >= 64 || !attr_set[dev]) {
        e = cudaFuncSetAttribute(decode_gqa_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)smem);
        if (e != cudaSuccess) return e;
        if (dev >= 0 && dev < 64) attr_set[dev] = true;
      }
    }
    // Longer splits than the per-head plan (each CTA now serves up to 16 heads):
    // double while there are still ~8 CTAs per SM.  Fewer splits use less of
    // the caller's workspace, laid out with the same stride rule.
    DecodeParams q = p;
    const long long pairs = (long long)p.num_seqs * p.H_kv * n_hg;
    while (q.split_tokens < 4096 && q.split_tokens * 2 <= kMaxSplitPages * q.page_size &&
           pairs * ((p.max_seq_len + 2LL * q.split_tokens - 1) / (2LL * q.split_tokens)) >=
               148LL * kGqaCtasPerSm)
      q.split_tokens *= 2;
    q.max_splits = (p.max_seq_len + q.split_tokens - 1) / q.split_tokens;
    dim3 grid(q.max_splits, p.H_kv * n_hg, p.num_seqs);
    decode_gqa_kernel<<<grid, kGqaThreads, smem, stream>>>(q);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    return q.max_splits > 1 ? launch_combine(q, stream) : cudaSuccess;
  } else {
    dim3 grid(p.max_splits, p.H, p.num_seqs);
    decode_split_kernel<4><<<grid, kThreads, 0, stream>>>(p);
  }
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (p.max_splits > 1) {
    combine_kernel<<<dim3(p.H, p.num_seqs), D, 0, stream>>>(p);
    e = cudaGetLastError();
  }
  return e;
}

}  // namespace pkv
