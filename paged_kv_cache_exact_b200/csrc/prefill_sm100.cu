// Tensor-core attention prefill for sm_100a (bf16 in/out, f32 accumulation).
//
// The method is the tiled online softmax of "Flash Attention: Fast,
// Memory-Efficient Attention for LLMs", section "The Algorithm": for each K/V
// tile, S = Q K^T, a running row max m and row sum l, P = exp(S - m), and the
// output accumulator rescaled when m moves; S and P never leave the SM.  Its
// "Flash Attention 2" section's causal skip is kept (tiles past the diagonal
// are never loaded).  K/V come either from contiguous [B, H_kv, N, d] tensors
// or, for paged prefill, straight from the pages through the block table
// ("What is Paged FlashAttention?", "How does it work?"), one TMA box per page.
//
// The B200 design (the pages' H100/SRAM tiling is prior art only):
//
// * CTA = two 128-row Q tiles of one (batch, head) sharing every K/V tile.
//   Warp roles: warps 0-3 and 4-7 are the softmax warpgroups of Q tile 0 and 1
//   (one thread per row = one TMEM lane), warp 8 issues TMA loads, warp 9
//   issues tcgen05.mma from one elected lane, warps 10-11 only lend registers.
// * TMEM (512 columns x 128 lanes x 32 bit): S0 | S1 | O0 | O1, 128 f32 columns
//   each.  P (bf16) overwrites the first 64 columns of its S once the softmax
//   has read S into registers, and feeds the PV product straight from TMEM
//   (A operand in tensor memory), so P never touches shared memory.
// * Shared memory: Q0, Q1 and a 2-stage ring for K and one for V, 32 KB per
//   128x128 bf16 tile, all in the 128-byte-swizzled K-major layout TMA writes.
// * Issue order on the MMA warp is S0(j+1) right after PV0(j) and S1(j+1)
//   right after PV1(j): while the softmax of one Q tile runs, the tensor core
//   works on the other tile (ping-pong).  tcgen05.mma executes in issue order,
//   so S_i(j+1) may overwrite P_i(j) once PV_i(j) has been issued.
// * Online softmax in base 2 with the scale folded into one FFMA; the output
//   is rescaled only when the running max grows by more than 2^8 (exact: O and
//   l always share the same reference max, and p stays <= 2^8).
// * Every mbarrier wait is bounded (about 2 s); on expiry the CTA records
//   PKV_DEVERR_TIMEOUT, stops issuing work, drains what it already issued and
//   frees its TMEM.
#include <cuda.h>

#include <mutex>

#include "common.cuh"
#include "exp2_poly.cuh"
#include "sm100_ptx.cuh"

namespace pkv {
namespace {

using namespace sm100;

constexpr int D = 128;             // head dim
constexpr int BM = 128;            // rows per Q tile
constexpr int BN = 128;            // keys per K/V tile
constexpr int kQTiles = 2;         // Q tiles per CTA
constexpr int kStages = 2;         // K ring and V ring depth
constexpr int kThreads = 384;      // 3 warpgroups: softmax 0, softmax 1, producer/MMA
// Register split: launched at kLaunchRegs per thread (3 warps per SM
// sub-partition -> at most 168), then the producer/MMA warpgroup drops to
// kRegsSide and both softmax warpgroups rise to kRegsSoftmax.  The split must
// add up to no more than the launch allocation or setmaxnreg.inc would wait
// forever, so the host refuses to launch unless the kernel was built with
// exactly kLaunchRegs registers.
constexpr int kLaunchRegs = 168;
constexpr int kRegsSoftmax = 208;
constexpr int kRegsSide = 88;
static_assert(2 * 128 * kRegsSoftmax + 128 * kRegsSide <= kThreads * kLaunchRegs,
              "register split exceeds the launch allocation");
constexpr int kTileBytes = BM * D * 2;             // 32 KB
constexpr int kHalfBytes = kTileBytes / 2;         // one 64-column block: 16 KB
constexpr uint64_t kWaitLimitNs = 2000000000ull;   // 2 s
constexpr float kRescaleThreshold = 8.0f;          // log2 units
// Softmax tuning: one exp2 pair in kPolyEvery goes to the FMA-pipe polynomial
// (0 = all on MUFU; measured slower at 1/8, 1/4 and 1/2, so off); kSplitP
// hands P to the PV product in two halves.
#ifndef PKV_POLY_EVERY
#define PKV_POLY_EVERY 0
#endif
#ifndef PKV_SPLIT_P
#define PKV_SPLIT_P 1
#endif
constexpr int kPolyEvery = PKV_POLY_EVERY;
// Start the first half's exponentials against the current reference max while
// the row max is reduced (redo rows whose max grew past the threshold).
// Measured: +2.5% on the 4x32x4096 prefill, -5..15% on the 32K paged prefill.
#ifndef PKV_SPEC_EXP
#define PKV_SPEC_EXP 0
#endif
constexpr bool kSpeculativeExp = PKV_SPEC_EXP != 0;
constexpr bool kSplitP = PKV_SPLIT_P != 0;

// Shared memory map (offsets from a 1024-aligned base).
constexpr int kOffQ = 0;
constexpr int kOffK = kOffQ + kQTiles * kTileBytes;
constexpr int kOffV = kOffK + kStages * kTileBytes;
constexpr int kOffBar = kOffV + kStages * kTileBytes;
enum Bar {
  kBarQ = 0,
  kBarKFull = 1,                      // + stage
  kBarKEmpty = kBarKFull + kStages,   // + stage
  kBarVFull = kBarKEmpty + kStages,
  kBarVEmpty = kBarVFull + kStages,
  kBarSFull = kBarVEmpty + kStages,   // + q tile
  kBarPHalf = kBarSFull + kQTiles,   // first 64 keys of P in TMEM (+ q tile)
  kBarPFull = kBarPHalf + kQTiles,    // all of P in TMEM
  kBarODone = kBarPFull + kQTiles,
  kBarVFixed = kBarODone + kQTiles,   // last paged V tile after tail rows are zeroed
  kBarDrain = kBarVFixed + 1,         // abort path: wait for issued MMAs
  kNumBars = kBarDrain + 1
};
constexpr int kOffTmemSlot = kOffBar + kNumBars * 8;
constexpr int kOffAbort = kOffTmemSlot + 4;
constexpr int kSmemUsed = kOffAbort + 4;
constexpr int kSmemBytes = kSmemUsed + 1024;       // slack for 1024-byte alignment

// TMEM columns.
constexpr uint32_t kColS = 0;      // + 128 * tile
constexpr uint32_t kColO = 256;    // + 128 * tile

constexpr uint32_t kIdescS = make_idesc_bf16(BM, BN, false);  // Q (K-major) x K (K-major)
constexpr uint32_t kIdescS8 = make_idesc_e4m3(BM, BN);         // e4m3 Q x e4m3 K
// e4m3 Q/K tiles: 128 rows of 128 one-byte elements, a single 128-byte-swizzled
// column block (16 KB) at the start of the same 32 KB slots the bf16 tiles use.
constexpr int kTileBytes8 = BM * D;
constexpr uint32_t kIdescO = make_idesc_bf16(BM, D, true);    // P (TMEM) x V (MN-major)

struct Geometry {
  int b, h, kvh, q0, q_len, kv_len, off, n_tiles;
};

__device__ __forceinline__ Geometry cta_geometry(const PrefillParams& p) {
  Geometry g;
  // 1-D grid, scheduled in groups of p.head_group (batch, head) pairs: within
  // a group the heaviest causal Q block of every head comes first, then the
  // next heaviest, ...  The host sizes a group so that its K/V (about 32 MB)
  // stays in L2 while its Q blocks run; the lightest blocks fill the tail.
  const int m_blocks = (p.q_len + BM * kQTiles - 1) / (BM * kQTiles);
  const int BH = p.B * p.H;
  const int hg = p.head_group;
  const int per_group = hg * m_blocks;
  const int group = blockIdx.x / per_group;
  const int r = blockIdx.x - group * per_group;
  const int heads_here = min(hg, BH - group * hg);
  const int rank = r / heads_here;                  // 0 = heaviest Q block
  const int bh = group * hg + (r - rank * heads_here);
  g.b = bh / p.H;
  g.h = bh % p.H;
  g.kvh = g.h / (p.H / p.H_kv);
  g.q0 = (m_blocks - 1 - rank) * (BM * kQTiles);
  g.q_len = p.q_len;
  int kv_len = p.kv_len;
  if (p.paged) {
    kv_len = p.seq_lens[g.b];
    const int cap = min(p.max_seq_len, p.max_pages * p.page_size);
    if (kv_len < p.q_len || kv_len > cap) {
      if (g.q0 == 0 && g.h == 0 && threadIdx.x == 0) flag_error(p.err, PKV_DEVERR_BAD_LEN);
      kv_len = max(0, min(kv_len, cap));
    }
  }
  g.kv_len = kv_len;
  g.off = kv_len - p.q_len;
  int n = (kv_len + BN - 1) / BN;
  if (p.causal) {
    const int last_row = min(g.q0 + BM * kQTiles - 1, p.q_len - 1);
    const int last_key = last_row + g.off;      // may be < 0: nothing visible
    n = last_key < 0 ? 0 : min(n, last_key / BN + 1);
  }
  g.n_tiles = max(n, 0);
  return g;
}

// ----------------------------------------------------------------------------
template <bool kPaged, bool kFp8QK>
__global__ void __launch_bounds__(kThreads, 1)
prefill_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
               const __grid_constant__ CUtensorMap tmV, const PrefillParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  auto bar = [&](int i) { return sbase + kOffBar + 8 * i; };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffAbort);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const Geometry g = cta_geometry(p);
  const int n = g.n_tiles;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kNumBars; ++i) {
      // P halves: one arrival per softmax thread; everything else: one arrival.
      const bool per_thread = (i >= kBarPHalf && i < kBarPFull + kQTiles);
      const uint32_t cnt = per_thread ? 128u : 1u;
      mbar_init(bar(i), cnt);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 9) {
    tmem_alloc(sbase + kOffTmemSlot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + kOffTmemSlot);

  auto fail = [&]() {
    *abort_flag = 1;
    flag_error(p.err, PKV_DEVERR_TIMEOUT);
  };
  // A phase that has already completed costs one try_wait; the abort flag (a
  // shared-memory read) is consulted only once the caller has to wait.
  auto wait = [&](int b, uint32_t parity) -> bool {
    if (mbar_try_wait(bar(b), parity)) return true;
    if (*abort_flag) return false;
    if (!mbar_wait_bounded(bar(b), parity, kWaitLimitNs)) {
      fail();
      return false;
    }
    return true;
  };

  if (warp >= 8) regs_decrease<kRegsSide>();

  if (warp == 8) {
    // ------------------------------------------------------------ producer --
    // The warp runs the loop converged.  Contiguous tiles and pages of >= 128
    // tokens take one TMA box per 64-column block, issued by lane 0; shorter
    // pages take one box per page per block, and lane i resolves page i of the
    // tile and issues its boxes, so the boxes of a tile are issued in parallel
    // (one thread issuing 16 of them per K or V tile could not keep ahead of
    // the tensor core).  Each table entry is read once and serves K and V.
    if (n > 0) {
      if (lane == 0) {
        prefetch_tmap(&tmQ);
        prefetch_tmap(&tmK);
        prefetch_tmap(&tmV);
        const int qc2 = g.b * p.H + g.h;
        mbar_arrive_expect_tx(bar(kBarQ), kQTiles * (kFp8QK ? kTileBytes8 : kTileBytes));
        for (int t = 0; t < kQTiles; ++t)
          for (int c = 0; c < (kFp8QK ? 1 : 2); ++c)
            tma_load_3d(sbase + kOffQ + t * kTileBytes + c * kHalfBytes, &tmQ, c * 64,
                        g.q0 + t * BM, qc2, bar(kBarQ));
      }
      auto wwait = [&](int b, uint32_t parity) -> bool {
        return __all_sync(0xffffffffu, wait(b, parity));
      };
      int last_k = -1, last_v = -1;                  // last tile whose K / V load was issued
      const int rows_per_box = kPaged ? min(p.page_size, BN) : BN;
      const bool box_per_page = kPaged && rows_per_box < BN;
      const int n_valid_pages = kPaged ? (g.kv_len + p.page_size - 1) >> p.page_shift : 0;
      const int32_t* trow = p.block_table + (size_t)g.b * p.max_pages;
      bool ok = true;
      for (int j = 0; j < n && ok; ++j) {
        const int st = j % kStages;
        const uint32_t ph = (j / kStages) & 1;
        const int k0 = j * BN;
        // boxes of this tile that hold tokens of the sequence (never past its last page)
        const int nbox = kPaged ? min(BN / rows_per_box, n_valid_pages - (k0 >> p.page_shift)) : 1;
        const uint32_t bytes = kPaged ? nbox * rows_per_box * 256 : kTileBytes;
        // this lane's box: first token row of its page slice in the pool
        const int mine = box_per_page ? lane : 0;
        int row = 0;
        if (kPaged && mine < nbox) {
          int phys = trow[(k0 + mine * rows_per_box) >> p.page_shift];
          if (phys < 0 || phys >= p.num_pages) {     // never read outside the pool
            flag_error(p.err, PKV_DEVERR_BAD_PAGE);
            phys = 0;
          }
          row = phys * p.page_size + ((k0 + mine * rows_per_box) & (p.page_size - 1));
        }
        const bool issues = box_per_page ? lane < nbox : lane == 0;
        ok = wwait(kBarKEmpty + st, ph ^ 1);
        if (!ok) break;
        if (lane == 0) mbar_arrive_expect_tx(bar(kBarKFull + st), kFp8QK ? kTileBytes8 : bytes);
        __syncwarp();
        if (issues) {
          for (int c = 0; c < (kFp8QK ? 1 : 2); ++c) {
            const uint32_t dst = sbase + kOffK + st * kTileBytes + c * kHalfBytes;
            if (kPaged)
              tma_load_3d(dst + mine * rows_per_box * 128, &tmK, c * 64, g.kvh, row, bar(kBarKFull + st));
            else
              tma_load_3d(dst, &tmK, c * 64, k0, g.b * p.H_kv + g.kvh, bar(kBarKFull + st));
          }
        }
        last_k = j;
        ok = wwait(kBarVEmpty + st, ph ^ 1);
        if (!ok) break;
        if (lane == 0) mbar_arrive_expect_tx(bar(kBarVFull + st), bytes);
        __syncwarp();
        if (issues) {
          for (int c = 0; c < 2; ++c) {
            const uint32_t dst = sbase + kOffV + st * kTileBytes + c * kHalfBytes;
            if (kPaged)
              tma_load_3d(dst + mine * rows_per_box * 128, &tmV, c * 64, g.kvh, row, bar(kBarVFull + st));
            else
              tma_load_3d(dst, &tmV, c * 64, k0, g.b * p.H_kv + g.kvh, bar(kBarVFull + st));
          }
        }
        last_v = j;
      }
      if (!ok && lane == 0) {
        // Drain loads already in flight before the CTA's shared memory goes away.
        for (int jj = max(0, last_k - 1); jj <= last_k; ++jj)
          mbar_wait_bounded(bar(kBarKFull + jj % kStages), (jj / kStages) & 1, kWaitLimitNs);
        for (int jj = max(0, last_v - 1); jj <= last_v; ++jj)
          mbar_wait_bounded(bar(kBarVFull + jj % kStages), (jj / kStages) & 1, kWaitLimitNs);
      }
    }
    // Paged, last tile partial: rows past kv_len (poisoned tails, unread pages)
    // must be zero in V, since P = 0 there but 0 * NaN is NaN.  The whole warp
    // zeroes them once the tile has landed, then releases it to the MMA warp.
    if (kPaged && n > 0) {
      const int j = n - 1;
      const int valid = g.kv_len - j * BN;
      if (valid < BN) {
        __syncwarp();
        const int st = j % kStages;
        bool ok = !*abort_flag;
        if (lane == 0 && ok) ok = mbar_wait_bounded(bar(kBarVFull + st), (j / kStages) & 1, kWaitLimitNs);
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        if (ok) {
          uint8_t* vt = smem + kOffV + st * kTileBytes;
          const int nrows = BN - valid;
          for (int idx = lane; idx < nrows * 16; idx += 32) {       // 16 x 16 B per row (2 blocks)
            const int r = valid + idx / 16, part = idx % 16;
            *reinterpret_cast<uint4*>(vt + (part / 8) * kHalfBytes + r * 128 + (part % 8) * 16) =
                make_uint4(0, 0, 0, 0);
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(bar(kBarVFixed));
        } else if (lane == 0) {
          fail();
        }
      }
    }
  } else if (warp == 9) {
    // ----------------------------------------------------------------- MMA --
    // Issue order per K/V tile j: PV0(j) S0(j+1) PV1(j) S1(j+1).  The softmax of
    // one Q tile then overlaps the other tile's MMAs (ping-pong), and each
    // S_t(j+1) is issued after PV_t(j), which consumes the P_t(j) it overwrites
    // (tcgen05.mma executes in issue order).  Descriptors are precomputed per
    // stage so that an issue costs one add and the MMA: a 128x128x16 MMA
    // retires in 64 cycles, less than a descriptor rebuild takes.  The warp
    // runs converged and one elected lane issues.
    auto wwait = [&](int b, uint32_t parity) -> bool {
      return __all_sync(0xffffffffu, wait(b, parity));
    };
    if (n > 0) {
      const bool last_fix = kPaged && (g.kv_len - (n - 1) * BN) < BN;
      const uint64_t dq0 = make_sdesc(sbase + kOffQ, 16, 1024);
      const uint64_t dq1 = make_sdesc(sbase + kOffQ + kTileBytes, 16, 1024);
      const uint64_t dk0 = make_sdesc(sbase + kOffK, 16, 1024);
      const uint64_t dk1 = make_sdesc(sbase + kOffK + kTileBytes, 16, 1024);
      const uint64_t dv0 = make_sdesc(sbase + kOffV, kHalfBytes, 1024);
      const uint64_t dv1 = make_sdesc(sbase + kOffV + kTileBytes, kHalfBytes, 1024);
      const bool leader = elect_one();
      auto issue_s = [&](int t, int j) {
        const uint64_t dk = (j % kStages) ? dk1 : dk0;
        const uint64_t dq = t ? dq1 : dq0;
        const uint32_t tS = tmem + kColS + 128 * t;
        if (leader) {
          if (kFp8QK) {
#pragma unroll
            for (int kk = 0; kk < D / 32; ++kk)     // K = 32 e4m3 (32 bytes) per MMA
              mma_ss_f8(tS, dq + ((kk * 32) >> 4), dk + ((kk * 32) >> 4), kIdescS8, kk > 0);
          } else {
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint64_t koff = ((kk / 4) * kHalfBytes + (kk % 4) * 32) >> 4;
              mma_ss(tS, dq + koff, dk + koff, kIdescS, kk > 0);
            }
          }
          mma_commit(bar(kBarSFull + t));
        }
        __syncwarp();
      };
      // O_t += P_t V over key steps [kk0, kk0 + 4): P arrives in two halves.
      auto issue_pv_half = [&](int t, int j, int kk0) {
        const uint64_t dv = (j % kStages) ? dv1 : dv0;
        const uint32_t tS = tmem + kColS + 128 * t;
        const uint32_t tO = tmem + kColO + 128 * t;
        if (leader) {
#pragma unroll
          for (int kk = kk0; kk < kk0 + BN / 32; ++kk)
            mma_ts(tO, tS + kk * 8, dv + ((kk * 16 * 128) >> 4), kIdescO,
                   (j > 0 || kk > 0) ? 1u : 0u);
        }
        __syncwarp();
      };
      // PV_t(j).  With want_k the next K tile is checked while the second half
      // of P is still being written, so that PV's second half and S_t(j+1)
      // issue back to back once P is complete.
      auto issue_pv = [&](int t, int j, bool want_k = false) -> bool {
        if (kSplitP) {
          if (!wwait(kBarPHalf + t, j & 1)) return false;
          tc_fence_after();
          issue_pv_half(t, j, 0);
        }
        if (want_k && !wwait(kBarKFull + (j + 1) % kStages, ((j + 1) / kStages) & 1)) return false;
        if (!wwait(kBarPFull + t, j & 1)) return false;
        tc_fence_after();
        if (!kSplitP) issue_pv_half(t, j, 0);
        issue_pv_half(t, j, BN / 32);
        if (leader) mma_commit(bar(kBarODone + t));
        __syncwarp();
        return true;
      };
      auto commit = [&](int b) {
        if (leader) mma_commit(bar(b));
        __syncwarp();
      };
      bool ok = wwait(kBarQ, 0) && wwait(kBarKFull + 0, 0);
      if (ok) {
        tc_fence_after();
        issue_s(0, 0);
        issue_s(1, 0);
        commit(kBarKEmpty + 0);
      }
      for (int j = 0; j < n && ok; ++j) {
        const int st = j % kStages;
        if (last_fix && j == n - 1)
          ok = wwait(kBarVFixed, 0);
        else
          ok = wwait(kBarVFull + st, (j / kStages) & 1);
        ok = ok && issue_pv(0, j, j + 1 < n);
        if (!ok) break;
        if (j + 1 < n) {
          tc_fence_after();
          issue_s(0, j + 1);
        }
        ok = issue_pv(1, j);
        if (!ok) break;
        commit(kBarVEmpty + st);
        if (j + 1 < n) {
          issue_s(1, j + 1);
          commit(kBarKEmpty + (j + 1) % kStages);
        }
      }
      if (!ok) {
        // Let every MMA already issued finish before TMEM is released.
        commit(kBarDrain);
        mbar_wait_bounded(bar(kBarDrain), 0, kWaitLimitNs);
      }
    }
  } else if (warp < 8) {
    // ------------------------------------------------------------- softmax --
    regs_increase<kRegsSoftmax>();
    const int t = warp >> 2;                         // Q tile of this warpgroup
    const int r = threadIdx.x & 127;                 // row in tile = TMEM lane
    const int row = g.q0 + t * BM + r;               // query row
    const uint32_t lane_addr = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + lane_addr + kColS + 128 * t;
    const uint32_t tO = tmem + lane_addr + kColO + 128 * t;
    const float c = p.scale_log2;
    const int limit = p.causal ? min(row + g.off, g.kv_len - 1) : g.kv_len - 1;

    float m_ref = -INFINITY, l = 0.f;
    bool ok = true;
    // tcgen05.ld/st are warp-collective: every branch around them is warp-uniform.
    for (int j = 0; j < n; ++j) {
      ok = wait(kBarSFull + t, j & 1);
      if (ok && j > 0) ok = wait(kBarODone + t, (j - 1) & 1);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      uint32_t s[128];
#pragma unroll
      for (int ch = 0; ch < 4; ++ch) {
        uint32_t (&sub)[32] = *reinterpret_cast<uint32_t(*)[32]>(&s[32 * ch]);
        tmem_ld32(tS + 32 * ch, sub);
      }
      tmem_wait_ld();
      const int k0 = j * BN;
      const bool masked = k0 + BN - 1 > limit;       // diagonal or tail tile
      if (masked) {
#pragma unroll
        for (int i = 0; i < 128; ++i)
          if (k0 + i > limit) s[i] = __float_as_uint(-INFINITY);
      }
      // row max: eight chains of 3-input max (dependency depth 8)
      float am[8];
#pragma unroll
      for (int a = 0; a < 8; ++a) am[a] = __uint_as_float(s[a]);
#pragma unroll
      for (int i = 8; i + 16 <= 128; i += 16) {        // elements 8 .. 119
#pragma unroll
        for (int a = 0; a < 8; ++a)
          am[a] = max3(am[a], __uint_as_float(s[i + 2 * a]), __uint_as_float(s[i + 2 * a + 1]));
      }
#pragma unroll
      for (int a = 0; a < 8; ++a) am[a] = fmaxf(am[a], __uint_as_float(s[120 + a]));   // 120 .. 127
      const float mx = max3(max3(am[0], am[1], am[2]), max3(am[3], am[4], am[5]),
                            fmaxf(am[6], am[7]));
      // The first half's exponentials are computed against the current
      // reference max while the row max above is still being reduced (the two
      // are independent, so they interleave); they are redone only in rows
      // whose max grew past the rescale threshold, which after the first tile
      // is rare.  Masked tiles stay on MUFU (exact zeros); elsewhere
      // kPolyEvery selects the share of pairs on the FMA-pipe polynomial.
      const bool poly = !__any_sync(0xffffffffu, masked);
      const uint64_t c2 = f2(c, c);
      uint64_t acc[4];
      auto exp_half = [&](int ch, float neg_m, uint32_t (&pk)[32]) {
        const uint64_t nm2 = f2(neg_m, neg_m);
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const int e = 64 * ch + 2 * i;
          const uint64_t x2 = fma2(f2(__uint_as_float(s[e]), __uint_as_float(s[e + 1])), c2, nm2);
          float p0, p1;
          if (kPolyEvery > 0 && poly && (i % (kPolyEvery > 0 ? kPolyEvery : 1)) == kPolyEvery - 1) {
            exp2_poly_pair(x2, p0, p1);
          } else {
            float x0, x1;
            unf2(x2, x0, x1);
            p0 = ex2(x0);
            p1 = ex2(x1);
          }
          acc[i & 3] = add2(acc[i & 3], f2(p0, p1));
          pk[i] = pack_bf16x2(p0, p1);
        }
      };
#pragma unroll
      for (int a = 0; a < 4; ++a) acc[a] = f2(0.f, 0.f);
      uint32_t pk[32];
      if (kSpeculativeExp) exp_half(0, (m_ref == -INFINITY) ? 0.f : -m_ref, pk);
      const float m_tile = mx * c;                  // running max in log2 units
      float alpha = 1.f;
      bool rescale = false;
      if (m_tile > m_ref + kRescaleThreshold || (m_ref == -INFINITY && m_tile != -INFINITY)) {
        alpha = ex2(m_ref - m_tile);               // m_ref = -inf -> 0
        m_ref = m_tile;
        rescale = true;
      }
      const float neg_m = (m_ref == -INFINITY) ? 0.f : -m_ref;
      if (!kSpeculativeExp) exp_half(0, neg_m, pk);
      if (__any_sync(0xffffffffu, rescale)) {
        if (kSpeculativeExp && rescale) {          // redo this row's first half
#pragma unroll
          for (int a = 0; a < 4; ++a) acc[a] = f2(0.f, 0.f);
          exp_half(0, neg_m, pk);
        }
        // O must be rescaled before PV(j) may start, i.e. before any P is handed over.
        if (j > 0) {                               // alpha = 1 in rows that keep m
#pragma unroll
          for (int ch = 0; ch < 4; ++ch) {
            uint32_t o[32];
            tmem_ld32(tO + 32 * ch, o);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
            tmem_st32(tO + 32 * ch, o);
          }
        }
      }
      tmem_st32(tS, pk);
      if (kSplitP) {                               // first half of P: PV(j) may start
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(bar(kBarPHalf + t));
      }
      exp_half(1, neg_m, pk);
      tmem_st32(tS + 32, pk);
      float s0, s1;
      unf2(add2(add2(acc[0], acc[1]), add2(acc[2], acc[3])), s0, s1);
      l = l * alpha + (s0 + s1);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar(kBarPFull + t));
    }
    if (ok && n > 0) ok = wait(kBarODone + t, (n - 1) & 1);
    ok = __all_sync(0xffffffffu, ok);
    if (ok) tc_fence_after();
    // Epilogue: O / l -> bf16 -> global (rows past q_len are not stored).
    const bool have_o = ok && n > 0;                 // warp-uniform
    const bool store = row < g.q_len;
    __nv_bfloat16* out = static_cast<__nv_bfloat16*>(p.O) +
                         (((size_t)g.b * p.H + g.h) * p.q_len + (store ? row : 0)) * D;
    const float inv = (have_o && l > 0.f) ? 1.f / l : 0.f;
#pragma unroll
    for (int ch = 0; ch < 4; ++ch) {
      uint32_t o[32];
      if (have_o) {
        tmem_ld32(tO + 32 * ch, o);
        tmem_wait_ld();
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) o[i] = 0u;
      }
      if (store) {
        uint4 packed[4];
        uint32_t* pw = reinterpret_cast<uint32_t*>(packed);
#pragma unroll
        for (int i = 0; i < 16; ++i)
          pw[i] = pack_bf16x2(__uint_as_float(o[2 * i]) * inv, __uint_as_float(o[2 * i + 1]) * inv);
        uint4* dst = reinterpret_cast<uint4*>(out + 32 * ch);
#pragma unroll
        for (int i = 0; i < 4; ++i) dst[i] = packed[i];
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ----------------------------------------------------------------- host side --
using EncodeFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                              const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                              const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                              CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeFn get_encode() {
  static EncodeFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeFn>(ptr);
  });
  return fn;
}

// 3-D map, 128-byte swizzle, box {128 bytes of d, box1, box2} (64 bf16 or 128 e4m3);
// out-of-range reads fill zeros.
bool encode_3d(CUtensorMap* m, const void* base, uint64_t d0, uint64_t d1, uint64_t d2,
               uint64_t stride1_bytes, uint64_t stride2_bytes, uint32_t box1, uint32_t box2,
               bool bytes = false) {
  EncodeFn enc = get_encode();
  if (!enc) return false;
  const cuuint64_t dims[3] = {d0, d1, d2};
  const cuuint64_t strides[2] = {stride1_bytes, stride2_bytes};
  const cuuint32_t box[3] = {bytes ? 128u : 64u, box1, box2};
  const cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, bytes ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
             const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

template <bool kPaged, bool kFp8QK>
cudaError_t set_smem_attr() {
  static int done[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && done[dev]) return cudaSuccess;
  // The in-kernel register split assumes this exact launch allocation.
  cudaFuncAttributes fa;
  cudaError_t e = cudaFuncGetAttributes(&fa, prefill_kernel<kPaged, kFp8QK>);
  if (e != cudaSuccess) return e;
  if (fa.numRegs != kLaunchRegs) return cudaErrorNotSupported;
  e = cudaFuncSetAttribute(prefill_kernel<kPaged, kFp8QK>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           kSmemBytes);
  if (e == cudaSuccess && dev >= 0 && dev < 64) done[dev] = 1;
  return e;
}

}  // namespace

cudaError_t launch_prefill_bf16(const PrefillParams& p, cudaStream_t stream) {
  if (p.d != D) return cudaErrorNotSupported;
  CUtensorMap tq, tk, tv;
  const uint64_t row_bytes = D * 2;
  const bool f8 = p.fp8_qk != 0;
  if (f8 && p.paged) return cudaErrorNotSupported;
  const uint64_t qk_row = f8 ? D : row_bytes;        // e4m3 Q/K rows are 128 bytes
  // Q: [B*H, q_len, d]
  if (!encode_3d(&tq, p.Q, D, p.q_len, (uint64_t)p.B * p.H, qk_row, qk_row * p.q_len, BM, 1, f8))
    return cudaErrorInvalidValue;
  if (p.paged) {
    // pages [P, ps, H_kv, d] viewed as [P*ps tokens, H_kv, d]; one box = one page's rows.
    const uint32_t rows = p.page_size < BN ? p.page_size : BN;
    const uint64_t tokens = (uint64_t)p.num_pages * p.page_size;
    if (!encode_3d(&tk, p.K, D, p.H_kv, tokens, row_bytes, row_bytes * p.H_kv, 1, rows) ||
        !encode_3d(&tv, p.V, D, p.H_kv, tokens, row_bytes, row_bytes * p.H_kv, 1, rows))
      return cudaErrorInvalidValue;
  } else {
    const uint64_t bhkv = (uint64_t)p.B * p.H_kv;
    if (!encode_3d(&tk, p.K, D, p.kv_len, bhkv, qk_row, qk_row * p.kv_len, BN, 1, f8) ||
        !encode_3d(&tv, p.V, D, p.kv_len, bhkv, row_bytes, row_bytes * p.kv_len, BN, 1))
      return cudaErrorInvalidValue;
  }
  const long long m_blocks = (p.q_len + BM * kQTiles - 1) / (BM * kQTiles);
  const long long ctas = m_blocks * p.B * p.H;
  if (ctas > 0x7fffffffLL) return cudaErrorNotSupported;
  dim3 grid((unsigned)ctas);
  // Heads scheduled together: as many as keep about 32 MB of K/V live in L2
  // (query heads sharing a kv head count once).
  PrefillParams q = p;
  {
    const long long kv_len = p.paged ? p.max_seq_len : p.kv_len;
    const long long kv_bytes = 2LL * kv_len * D * 2;              // K and V of one kv head
    const int group_q = p.H / p.H_kv;
    long long hg = (32LL << 20) / (kv_bytes > 0 ? kv_bytes : 1) * group_q;
    hg = hg < 1 ? 1 : (hg > 32 ? 32 : hg);
    q.head_group = (int)hg;
  }
  cudaError_t e;
  if (p.paged) {
    e = set_smem_attr<true, false>();
    if (e != cudaSuccess) return e;
    prefill_kernel<true, false><<<grid, kThreads, kSmemBytes, stream>>>(tq, tk, tv, q);
  } else if (f8) {
    e = set_smem_attr<false, true>();
    if (e != cudaSuccess) return e;
    prefill_kernel<false, true><<<grid, kThreads, kSmemBytes, stream>>>(tq, tk, tv, q);
  } else {
    e = set_smem_attr<false, false>();
    if (e != cudaSuccess) return e;
    prefill_kernel<false, false><<<grid, kThreads, kSmemBytes, stream>>>(tq, tk, tv, q);
  }
  return cudaGetLastError();
}

}  // namespace pkv
