// float32 attention on the FMA pipes (contiguous or paged K/V, any q_len).
//
// The tiled, online-softmax formulation of "Flash Attention: Fast,
// Memory-Efficient Attention for LLMs", section "The Algorithm", in plain
// float32 arithmetic: a CTA holds 32 query rows, streams 32-key tiles of K and
// V into shared memory (through the block table when paged, as "What is Paged
// FlashAttention?" describes, with no gather), and keeps per-row running
// (max, sum, O) in registers.  Four threads share a query row; thread `part`
// owns dims part, part + 4, part + 8, ... so that the four threads of a row
// hit four different shared-memory banks.  This is the float32 path: tensor
// cores would round the inputs (TF32), so it stays on exact float32 FMAs.
#include "common.cuh"

namespace pkv {
namespace {

constexpr int kRows = 32;       // query rows per CTA
constexpr int kKeys = 32;       // keys per shared-memory tile
constexpr int kThreads = kRows * 4;

template <int D>
__global__ void __launch_bounds__(kThreads)
simt_f32_kernel(const SimtParams p) {
  constexpr int DP = D / 4;  // dims per thread
  __shared__ float sK[kKeys][D];
  __shared__ float sV[kKeys][D];
  __shared__ int s_phys[kKeys];

  const int b = blockIdx.z, h = blockIdx.y;
  const int tid = threadIdx.x;
  const int r = tid >> 2, part = tid & 3;
  const int row = blockIdx.x * kRows + r;
  const int kvh = h / (p.H / p.H_kv);

  int kv_len = p.kv_len;
  if (p.paged) {
    kv_len = p.seq_lens[b];
    const int cap = min(p.max_seq_len, p.max_pages * p.page_size);
    if (kv_len < p.q_len || kv_len > cap) {
      if (blockIdx.x == 0 && h == 0 && tid == 0) flag_error(p.err, PKV_DEVERR_BAD_LEN);
      kv_len = max(0, min(kv_len, cap));
    }
  }
  const int off = kv_len - p.q_len;     // causal: key j visible iff j <= i + off

  const size_t qrow = ((size_t)b * p.H + h) * p.q_len + row;
  float qf[DP], acc[DP];
#pragma unroll
  for (int i = 0; i < DP; ++i) {
    qf[i] = row < p.q_len ? p.q[qrow * D + part + 4 * i] * p.scale_log2 : 0.f;
    acc[i] = 0.f;
  }
  float m = -INFINITY, l = 0.f;

  // Keys this CTA needs: up to the last visible key of its last row.
  int last_row = min(blockIdx.x * kRows + kRows - 1, p.q_len - 1);
  int n_keys = p.causal ? min(kv_len, last_row + off + 1) : kv_len;
  n_keys = max(n_keys, 0);

  const float* kc = p.k;
  const float* vc = p.v;
  if (!p.paged) {
    kc += ((size_t)b * p.H_kv + kvh) * (size_t)p.kv_len * D;
    vc += ((size_t)b * p.H_kv + kvh) * (size_t)p.kv_len * D;
  }

  for (int j0 = 0; j0 < n_keys; j0 += kKeys) {
    __syncthreads();   // previous tile fully consumed
    if (p.paged && tid < kKeys) {
      const int t = j0 + tid;
      int phys = -1;
      if (t < n_keys) {
        phys = p.block_table[(size_t)b * p.max_pages + (t >> p.page_shift)];
        if (phys < 0 || phys >= p.num_pages) {
          flag_error(p.err, PKV_DEVERR_BAD_PAGE);
          phys = -1;
        }
      }
      s_phys[tid] = phys;
    }
    if (p.paged) __syncthreads();
    // Cooperative tile load: kKeys rows x D floats, as float4.
    for (int idx = tid; idx < kKeys * D / 4; idx += kThreads) {
      const int kr = idx / (D / 4), c4 = idx % (D / 4);
      const int t = j0 + kr;
      float4 kk = make_float4(0.f, 0.f, 0.f, 0.f), vv = kk;
      const float* ksrc = nullptr;
      const float* vsrc = nullptr;
      if (t < n_keys) {
        if (p.paged) {
          const int phys = s_phys[kr];
          if (phys >= 0) {
            const size_t tok = ((size_t)phys << p.page_shift) + (t & (p.page_size - 1));
            ksrc = p.k + (tok * p.H_kv + kvh) * D;
            vsrc = p.v + (tok * p.H_kv + kvh) * D;
          }
        } else {
          ksrc = kc + (size_t)t * D;
          vsrc = vc + (size_t)t * D;
        }
      }
      if (ksrc) {
        kk = reinterpret_cast<const float4*>(ksrc)[c4];
        vv = reinterpret_cast<const float4*>(vsrc)[c4];
      }
      reinterpret_cast<float4*>(&sK[kr][0])[c4] = kk;
      reinterpret_cast<float4*>(&sV[kr][0])[c4] = vv;
    }
    __syncthreads();

    float sc[kKeys];
    float mx = -INFINITY;
#pragma unroll
    for (int j = 0; j < kKeys; ++j) {
      float dot = 0.f;
#pragma unroll
      for (int i = 0; i < DP; ++i) dot = fmaf(qf[i], sK[j][part + 4 * i], dot);
      dot += __shfl_xor_sync(0xffffffffu, dot, 1);
      dot += __shfl_xor_sync(0xffffffffu, dot, 2);
      const int t = j0 + j;
      bool vis = t < n_keys && (!p.paged || s_phys[j] >= 0);
      if (p.causal) vis = vis && t <= row + off;
      sc[j] = vis ? dot : -INFINITY;
      mx = fmaxf(mx, sc[j]);
    }
    const float m_new = fmaxf(m, mx);
    if (m_new != -INFINITY) {
      const float alpha = ex2(m - m_new);
      l *= alpha;
#pragma unroll
      for (int i = 0; i < DP; ++i) acc[i] *= alpha;
#pragma unroll
      for (int j = 0; j < kKeys; ++j) {
        const float pr = ex2(sc[j] - m_new);
        l += pr;
#pragma unroll
        for (int i = 0; i < DP; ++i) acc[i] = fmaf(pr, sV[j][part + 4 * i], acc[i]);
      }
      m = m_new;
    }
  }

  if (row < p.q_len) {
    const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
    for (int i = 0; i < DP; ++i) p.out[qrow * D + part + 4 * i] = acc[i] * inv;
  }
}

}  // namespace

cudaError_t launch_simt_f32(const SimtParams& p, cudaStream_t stream) {
  dim3 grid((p.q_len + kRows - 1) / kRows, p.H, p.B);
  if (p.d == 64)
    simt_f32_kernel<64><<<grid, kThreads, 0, stream>>>(p);
  else
    simt_f32_kernel<128><<<grid, kThreads, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace pkv
