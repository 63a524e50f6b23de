// Tensor-core attention prefill for sm_100a (bf16 in/out, f32 accumulation).
//
// The method is the tiled online softmax of "Flash Attention: Fast,
// Memory-Efficient Attention for LLMs", section "The Algorithm": for each K/V
// tile, S = Q K^T, a running row max m and row sum l, P = exp(S - m), and the
// output accumulator rescaled when m moves; S and P never leave the SM.  Its
// "Flash Attention 2" section's causal skip is kept (tiles past the diagonal
// are never loaded, per Q tile).  K/V come either from contiguous
// [B, H_kv, N, d] tensors or, for paged prefill, straight from the pages
// through the block table ("What is Paged FlashAttention?", "How does it
// work?"), one TMA box per page.
//
// The B200 design (the pages' H100/SRAM tiling is prior art only):
//
// * Work item = two 128-row Q tiles of one (batch, head) sharing every K/V
//   tile.  The kernel is persistent: it is launched with one CTA per work
//   item, and a running CTA that nears the end of its item claims the next
//   unstarted CTA's item through cluster launch control (the hardware cancels
//   that CTA's launch and hands over its index).  Items keep their launch
//   order (heaviest causal blocks first, heads grouped for L2), the balance
//   stays that of the hardware's own greedy placement, and one item's tail
//   (last PV, epilogue) overlaps the next item's first loads and MMAs
//   instead of a CTA teardown and launch.
// * Warp roles: warps 0-3 and 4-7 are the softmax warpgroups of Q tile 0 and
//   1 (one thread per row = one TMEM lane; each also writes its tile's
//   output), warp 8 loads (TMA) and claims items, warp 9 issues tcgen05.mma
//   from one elected lane, warps 10-11 only lend registers.
// * TMEM (512 columns x 128 lanes x 32 bit): S0 | S1 | O0 | O1, 128 f32 columns
//   each.  P (bf16) overwrites the first 64 columns of its S once the softmax
//   has read S into registers, and feeds the PV product straight from TMEM
//   (A operand in tensor memory), so P never touches shared memory.
// * Shared memory: Q0, Q1 and a 2-stage ring for K and one for V, 32 KB per
//   128x128 bf16 tile, all in the 128-byte-swizzled K-major layout TMA writes.
// * Issue order on the MMA warp is S0(j+1) right after PV0(j) and S1(j+1)
//   right after PV1(j): while the softmax of one Q tile runs, the tensor core
//   works on the other tile (ping-pong).  tcgen05.mma executes in issue order,
//   so S_i(j+1) may overwrite P_i(j) once PV_i(j) has been issued, and the
//   next item's S_i(0) may follow this item's last PV_i at once.
// * Online softmax in base 2 with the scale folded into one FFMA; the output
//   is rescaled only when the running max grows by more than 2^8 (exact: O and
//   l always share the same reference max, and p stays <= 2^8).
// * Every mbarrier wait is bounded; on expiry the CTA records
//   PKV_DEVERR_TIMEOUT, every role stops, drains what it already issued (TMA
//   loads, MMAs, an item claim) and the CTA frees its TMEM and exits.
// * A page id outside the pool is never read: its keys are left out of the
//   softmax (as the decode kernel does) and its V rows are zeroed, and
//   PKV_DEVERR_BAD_PAGE is recorded.
#include <cuda.h>

#include <mutex>

#include "common.cuh"
#include "sm100_ptx.cuh"

namespace pkv {
namespace {

using namespace sm100;

constexpr int D = 128;             // head dim
constexpr int BM = 128;            // rows per Q tile
constexpr int BN = 128;            // keys per K/V tile
constexpr int kQTiles = 2;         // Q tiles per work item
constexpr int kStages = 2;         // K ring and V ring depth
constexpr int kThreads = 384;      // 3 warpgroups: softmax 0, softmax 1, loader/MMA
// Register split: launched at kLaunchRegs per thread (3 warps per SM
// sub-partition -> at most 168), then the loader/MMA warpgroup drops to
// kRegsSide and both softmax warpgroups rise to kRegsSoftmax.  The split must
// add up to no more than the launch allocation or setmaxnreg.inc would wait
// forever, so the build fails unless the kernel compiles to exactly
// kLaunchRegs registers.
constexpr int kLaunchRegs = 168;
constexpr int kRegsSoftmax = 208;
constexpr int kRegsSide = 88;
static_assert(2 * 128 * kRegsSoftmax + 128 * kRegsSide <= kThreads * kLaunchRegs,
              "register split exceeds the launch allocation");
constexpr int kTileBytes = BM * D * 2;             // 32 KB
constexpr int kHalfBytes = kTileBytes / 2;         // one 64-column block: 16 KB
constexpr uint64_t kDefaultWaitNs = 2000000000ull; // 2 s
constexpr float kRescaleThreshold = 8.0f;          // log2 units
constexpr int kMaskSlots = 4;      // bad-page masks of the K/V tiles in flight
constexpr int kClaimLead = 3;      // claim the next item this many K/V tiles before the last
constexpr int kItemReaders = 9;    // warps that read a claimed item id: 8 softmax + MMA

// Shared memory map (offsets from a 1024-aligned base).
constexpr int kOffQ = 0;
constexpr int kOffK = kOffQ + kQTiles * kTileBytes;
constexpr int kOffV = kOffK + kStages * kTileBytes;
constexpr int kOffBar = kOffV + kStages * kTileBytes;
enum Bar {
  kBarQFull = 0,                      // + q tile
  kBarQEmpty = kBarQFull + kQTiles,   // + q tile: the item's last S_t has run
  kBarKFull = kBarQEmpty + kQTiles,   // + stage
  kBarKEmpty = kBarKFull + kStages,   // + stage
  kBarVFull = kBarKEmpty + kStages,
  kBarVEmpty = kBarVFull + kStages,
  kBarSFull = kBarVEmpty + kStages,   // + q tile
  kBarPHalf = kBarSFull + kQTiles,    // first 64 keys of P in TMEM (+ q tile)
  kBarPFull = kBarPHalf + kQTiles,    // all of P in TMEM
  kBarODone = kBarPFull + kQTiles,
  kBarVFixed = kBarODone + kQTiles,   // last paged V tile after tail rows are zeroed
  kBarItem = kBarVFixed + 1,          // + slot: a claimed item id is published
  kBarItemFree = kBarItem + 2,        // + slot: every reader has taken it
  kBarClaim = kBarItemFree + 2,       // a launch-control response landed
  kBarDrain = kBarClaim + 1,          // abort path: wait for issued MMAs
  kNumBars = kBarDrain + 1
};
constexpr int kOffClaim = (kOffBar + kNumBars * 8 + 15) & ~15;   // 16-byte response
constexpr int kOffItem = kOffClaim + 16;                         // int[2]
constexpr int kOffMask = kOffItem + 8;                           // uint32[kMaskSlots]
constexpr int kOffTmemSlot = kOffMask + 4 * kMaskSlots;
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

// A bad-page mask slot holds the K/V tile's running index (low 24 bits) in
// bits 8..31 and one bit per page box of the tile (at most 8) in bits 0..7.
PKV_DEVINLINE uint32_t mask_word(int kv_index, uint32_t bits) {
  return (static_cast<uint32_t>(kv_index & 0xFFFFFF) << 8) | bits;
}

struct Geometry {
  int b, h, kvh, q0, kv_len, off;
  int n[kQTiles];   // K/V tiles Q tile t needs (0: the tile has no rows)
  int nmax;         // K/V tiles the item loads
  bool bad_len;
};

// Work item `item` of the launch order: groups of p.head_group (batch, head)
// pairs; within a group the heaviest causal Q block of every head comes
// first, then the next heaviest, ...  The host sizes a group so that its K/V
// (about 64 MB) stays in L2 while its Q blocks run.
__device__ __forceinline__ Geometry item_geometry(const PrefillParams& p, int item) {
  Geometry g;
  const int m_blocks = (p.q_len + BM * kQTiles - 1) / (BM * kQTiles);
  const int BH = p.B * p.H;
  const int hg = p.head_group;
  const int per_group = hg * m_blocks;
  const int group = item / per_group;
  const int r = item - group * per_group;
  const int heads_here = min(hg, BH - group * hg);
  const int rank = r / heads_here;                  // 0 = heaviest Q block
  const int bh = group * hg + (r - rank * heads_here);
  g.b = bh / p.H;
  g.h = bh % p.H;
  g.kvh = g.h / (p.H / p.H_kv);
  g.q0 = (m_blocks - 1 - rank) * (BM * kQTiles);
  int kv_len = p.kv_len;
  g.bad_len = false;
  if (p.paged) {
    kv_len = p.seq_lens[g.b];
    const int cap = min(p.max_seq_len, p.max_pages * p.page_size);
    if (kv_len < p.q_len || kv_len > cap) {
      g.bad_len = true;
      kv_len = max(0, min(kv_len, cap));
    }
  }
  g.kv_len = kv_len;
  g.off = kv_len - p.q_len;
  const int n_kv = (kv_len + BN - 1) / BN;
  g.nmax = 0;
#pragma unroll
  for (int t = 0; t < kQTiles; ++t) {
    const int first = g.q0 + t * BM;
    int n = 0;
    if (first < p.q_len) {
      n = n_kv;
      if (p.causal) {
        const int last_key = min(first + BM - 1, p.q_len - 1) + g.off;   // < 0: nothing visible
        n = last_key < 0 ? 0 : min(n_kv, last_key / BN + 1);
      }
    }
    g.n[t] = n;
    g.nmax = max(g.nmax, n);
  }
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
  volatile int* item_slot = reinterpret_cast<volatile int*>(smem + kOffItem);
  volatile uint32_t* mask_slot = reinterpret_cast<volatile uint32_t*>(smem + kOffMask);
  const uint64_t limit_ns = p.wait_limit_ns ? p.wait_limit_ns : kDefaultWaitNs;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kNumBars; ++i) {
      uint32_t cnt = 1;
      if (i >= kBarPHalf && i < kBarPFull + kQTiles) cnt = 128;   // one arrival per softmax thread
      if (i >= kBarItemFree && i < kBarItemFree + 2) cnt = kItemReaders;
      mbar_init(bar(i), cnt);
    }
    for (int s = 0; s < kMaskSlots; ++s) mask_slot[s] = mask_word(s - kMaskSlots, 0);
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
    if (!*abort_flag) {
      *abort_flag = 1;
      flag_error(p.err, PKV_DEVERR_TIMEOUT);
    }
  };
  // A phase that has already completed costs one try_wait; the abort flag (a
  // shared-memory read) is consulted only once the caller has to wait.
  auto wait = [&](int b, uint32_t parity) -> bool {
    if (mbar_try_wait(bar(b), parity)) return true;
    if (*abort_flag) return false;
    if (!mbar_wait_abortable(bar(b), parity, limit_ns, abort_flag)) {
      fail();
      return false;
    }
    return true;
  };
  auto wwait = [&](int b, uint32_t parity) -> bool {   // warp-uniform result
    return __all_sync(0xffffffffu, wait(b, parity));
  };
  // Item id number `kk` claimed after the CTA's own (a whole warp calls this):
  // wait until the loader publishes it, read it, and release the slot.  -1 =
  // no item left; -2 = the CTA is aborting.
  auto read_item = [&](int kk) -> int {
    if (!wwait(kBarItem + (kk & 1), (kk >> 1) & 1)) return -2;
    const int v = item_slot[kk & 1];
    __syncwarp();
    if (lane == 0) mbar_arrive(bar(kBarItemFree + (kk & 1)));
    return v;
  };

  if (warp >= 8) regs_decrease<kRegsSide>();

  if (warp == 8) {
    // ------------------------------------------------------------- loader --
    // The warp runs converged.  Contiguous tiles and pages of >= 128 tokens
    // take one TMA box per 64-column block, issued by lane 0; shorter pages
    // take one box per page per block, and lane i resolves page i of the tile
    // and issues its boxes, so the boxes of a tile are issued in parallel.
    // Each table entry is read once and serves K and V.
    if (lane == 0) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
    }
    const uint32_t qk_bytes = kFp8QK ? kTileBytes8 : kTileBytes;
    const int rows_per_box = kPaged ? min(p.page_size, BN) : BN;
    const bool box_per_page = kPaged && rows_per_box < BN;
    int kv_it = 0, tail_it = 0, claims = 0;
    int q_it[kQTiles] = {0, 0};
    // Loads issued whose completion nobody has seen yet (for the abort
    // drain), two bits per barrier: bit 0 = pending, bit 1 = its phase parity.
    // Fields: K stage s at 2s, V stage s at 4 + 2s, Q tile t at 8 + 2t.
    uint32_t pend = 0;
    auto set_pend = [&](int field, uint32_t parity) {
      pend = (pend & ~(3u << (2 * field))) | ((1u | (parity << 1)) << (2 * field));
    };
    auto clear_pend = [&](int field) { pend &= ~(3u << (2 * field)); };
    bool pend_claim = false;
    bool claim_live = true;     // after a failed claim no further claim may be made
    bool ok = true;
    int item = blockIdx.x;
    for (int k = 0; ok && item >= 0; ++k) {
      const Geometry g = item_geometry(p, item);
      if (g.bad_len && g.q0 == 0 && g.h == 0 && lane == 0) flag_error(p.err, PKV_DEVERR_BAD_LEN);
      const int nmax = g.nmax;
      bool claimed = false;
      auto claim = [&]() {
        if (lane == 0) {
          mbar_arrive_expect_tx(bar(kBarClaim), 16);
          clc_try_cancel(sbase + kOffClaim, bar(kBarClaim));
        }
        __syncwarp();
        claimed = true;
        pend_claim = true;
      };
      auto load_q = [&](int t) -> bool {
        if (!wwait(kBarQEmpty + t, (q_it[t] & 1) ^ 1)) return false;
        if (lane == 0) {
          mbar_arrive_expect_tx(bar(kBarQFull + t), qk_bytes);
          for (int c = 0; c < (kFp8QK ? 1 : 2); ++c)
            tma_load_3d(sbase + kOffQ + t * kTileBytes + c * kHalfBytes, &tmQ, c * 64,
                        g.q0 + t * BM, g.b * p.H + g.h, bar(kBarQFull + t));
        }
        __syncwarp();
        set_pend(4 + t, q_it[t] & 1);
        return true;
      };
      if (g.n[0] > 0) ok = load_q(0);
      const int n_valid_pages = kPaged ? (g.kv_len + p.page_size - 1) >> p.page_shift : 0;
      const int32_t* trow = p.block_table + (size_t)g.b * p.max_pages;
      for (int j = 0; j < nmax && ok; ++j) {
        if (!claimed && claim_live && j >= nmax - kClaimLead) claim();
        const int it = kv_it + j;
        const int st = it % kStages;
        const uint32_t ph = (it / kStages) & 1;
        const int k0 = j * BN;
        // boxes of this tile that hold tokens of the sequence (never past its last page)
        const int nbox = kPaged ? min(BN / rows_per_box, n_valid_pages - (k0 >> p.page_shift)) : 1;
        const int mine = box_per_page ? lane : 0;     // this lane's box
        int row = 0;
        bool good = true;
        if (kPaged && mine < nbox) {
          const int phys = trow[(k0 + mine * rows_per_box) >> p.page_shift];
          good = phys >= 0 && phys < p.num_pages;     // never read outside the pool
          row = phys * p.page_size + ((k0 + mine * rows_per_box) & (p.page_size - 1));
        }
        const bool in_tile = box_per_page ? lane < nbox : lane == 0;
        const uint32_t bad = kPaged ? __ballot_sync(0xffffffffu, in_tile && !good) : 0u;
        // bad boxes: bit b = box b (box_per_page), or bit 0 = the whole tile
        const uint32_t bad_boxes = box_per_page ? bad : (bad ? 1u : 0u);
        const int n_good = (kPaged ? nbox : 1) - __popc(bad_boxes);
        const uint32_t bytes = kPaged ? n_good * rows_per_box * 256 : qk_bytes;
        const bool issues = in_tile && good;
        if (kPaged && bad && lane == 0) flag_error(p.err, PKV_DEVERR_BAD_PAGE);

        ok = wwait(kBarKEmpty + st, ph ^ 1);
        if (!ok) break;
        clear_pend(st);
        if (kPaged && lane == 0) mask_slot[it % kMaskSlots] = mask_word(it, bad_boxes);
        const bool stall = p.stall_tile_plus1 == j + 1 && k == 0;   // test hook: K(j) never lands
        if (lane == 0) mbar_arrive_expect_tx(bar(kBarKFull + st), kFp8QK ? kTileBytes8 : bytes);
        __syncwarp();
        if (issues && !stall) {
          for (int c = 0; c < (kFp8QK ? 1 : 2); ++c) {
            const uint32_t dst = sbase + kOffK + st * kTileBytes + c * kHalfBytes;
            if (kPaged)
              tma_load_3d(dst + mine * rows_per_box * 128, &tmK, c * 64, g.kvh, row, bar(kBarKFull + st));
            else
              tma_load_3d(dst, &tmK, c * 64, k0, g.b * p.H_kv + g.kvh, bar(kBarKFull + st));
          }
        }
        if (!stall && __any_sync(0xffffffffu, issues)) set_pend(st, ph);
        if (j == 0 && g.n[1] > 0) {
          ok = load_q(1);
          if (!ok) break;
        }

        ok = wwait(kBarVEmpty + st, ph ^ 1);
        if (!ok) break;
        clear_pend(2 + st);
        if (kPaged && bad_boxes) {
          // V rows of skipped boxes must be zero: P is 0 there, but 0 * NaN = NaN.
          uint8_t* vt = smem + kOffV + st * kTileBytes;
          for (int idx = lane; idx < BN * 16; idx += 32) {   // 16 x 16 B per row (2 blocks)
            const int r = idx / 16, part = idx % 16;
            if (!((bad_boxes >> (box_per_page ? r / rows_per_box : 0)) & 1)) continue;
            *reinterpret_cast<uint4*>(vt + (part / 8) * kHalfBytes + r * 128 + (part % 8) * 16) =
                make_uint4(0, 0, 0, 0);
          }
          fence_proxy_async_smem();
        }
        __syncwarp();
        if (lane == 0) mbar_arrive_expect_tx(bar(kBarVFull + st), kPaged ? bytes : kTileBytes);
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
        if (__any_sync(0xffffffffu, issues)) set_pend(2 + st, ph);
      }
      if (!ok) break;
      if (!claimed && claim_live) claim();
      // Paged, last tile partial: rows past kv_len (poisoned tails, unread
      // pages) must be zero in V, since P = 0 there but 0 * NaN is NaN.  The
      // whole warp zeroes them once the tile has landed, then releases it to
      // the MMA warp.
      if (kPaged && nmax > 0 && g.kv_len - (nmax - 1) * BN < BN) {
        const int it = kv_it + nmax - 1;
        const int st = it % kStages;
        const int valid = g.kv_len - (nmax - 1) * BN;
        if ((pend >> (2 * (2 + st))) & 1) ok = wwait(kBarVFull + st, (it / kStages) & 1);
        if (!ok) break;
        clear_pend(2 + st);
        uint8_t* vt = smem + kOffV + st * kTileBytes;
        for (int idx = lane; idx < (BN - valid) * 16; idx += 32) {   // 16 x 16 B per row
          const int r = valid + idx / 16, part = idx % 16;
          *reinterpret_cast<uint4*>(vt + (part / 8) * kHalfBytes + r * 128 + (part % 8) * 16) =
              make_uint4(0, 0, 0, 0);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(kBarVFixed));
        ++tail_it;
      }
      // The next item: the one the claim returned, or none.
      int next = -1;
      if (claim_live) {
        ok = wwait(kBarClaim, claims & 1);
        if (!ok) break;
        pend_claim = false;
        ++claims;
        next = __shfl_sync(0xffffffffu, lane == 0 ? clc_cancelled_x(sbase + kOffClaim) : 0, 0);
        if (next < 0) claim_live = false;
      }
      ok = wwait(kBarItemFree + (k & 1), ((k >> 1) & 1) ^ 1);
      if (!ok) break;
      if (lane == 0) {
        item_slot[k & 1] = next;
        mbar_arrive(bar(kBarItem + (k & 1)));
      }
      __syncwarp();
      kv_it += nmax;
#pragma unroll
      for (int t = 0; t < kQTiles; ++t) q_it[t] += g.n[t] > 0;
      item = next;
    }
    if (!ok && lane == 0) {
      // Drain loads (and a claim) in flight before the CTA's shared memory goes away.
      // field f: barrier kBarKFull + s (f = s), kBarVFull + s (f = 2 + s) or
      // kBarQFull + t (f = 4 + t)
      const int field_bar[6] = {kBarKFull, kBarKFull + 1, kBarVFull, kBarVFull + 1, kBarQFull,
                                kBarQFull + 1};
      for (int f = 0; f < 6; ++f)
        if ((pend >> (2 * f)) & 1)
          mbar_wait_bounded(bar(field_bar[f]), (pend >> (2 * f + 1)) & 1, limit_ns);
      if (pend_claim) mbar_wait_bounded(bar(kBarClaim), claims & 1, limit_ns);
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
    const uint64_t dq[kQTiles] = {make_sdesc(sbase + kOffQ, 16, 1024),
                                  make_sdesc(sbase + kOffQ + kTileBytes, 16, 1024)};
    const uint64_t dk0 = make_sdesc(sbase + kOffK, 16, 1024);
    const uint64_t dk1 = make_sdesc(sbase + kOffK + kTileBytes, 16, 1024);
    const uint64_t dv0 = make_sdesc(sbase + kOffV, kHalfBytes, 1024);
    const uint64_t dv1 = make_sdesc(sbase + kOffV + kTileBytes, kHalfBytes, 1024);
    const bool leader = elect_one();
    int kv_it = 0, tail_it = 0;
    int q_it[kQTiles] = {0, 0}, p_it[kQTiles] = {0, 0};
    bool ok = true;
    for (int k = 0; ok; ++k) {
      const int item = k == 0 ? blockIdx.x : read_item(k - 1);
      if (item == -2) ok = false;
      if (item < 0) break;
      const Geometry g = item_geometry(p, item);
      const int nmax = g.nmax;
      if (nmax == 0) continue;
      const bool last_fix = kPaged && g.kv_len - (nmax - 1) * BN < BN;
      int s_left[kQTiles] = {g.n[0], g.n[1]};
      auto commit = [&](int b) {
        if (leader) mma_commit(bar(b));
        __syncwarp();
      };
      // S_t = Q_t K(j)^T for K/V tile j of this item (K(j) has landed).
      auto issue_s = [&](int t, int j) {
        const uint64_t dk = ((kv_it + j) % kStages) ? dk1 : dk0;
        const uint32_t tS = tmem + kColS + 128 * t;
        if (leader) {
          if (kFp8QK) {
#pragma unroll
            for (int kk = 0; kk < D / 32; ++kk)     // K = 32 e4m3 (32 bytes) per MMA
              mma_ss_f8(tS, dq[t] + ((kk * 32) >> 4), dk + ((kk * 32) >> 4), kIdescS8, kk > 0);
          } else {
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint64_t koff = ((kk / 4) * kHalfBytes + (kk % 4) * 32) >> 4;
              mma_ss(tS, dq[t] + koff, dk + koff, kIdescS, kk > 0);
            }
          }
          mma_commit(bar(kBarSFull + t));
          if (--s_left[t] == 0) mma_commit(bar(kBarQEmpty + t));   // Q_t may be reloaded
        }
        __syncwarp();
      };
      // O_t += P_t V over key steps [kk0, kk0 + 4): P arrives in two halves.
      auto issue_pv_half = [&](int t, int j, int kk0) {
        const uint64_t dv = ((kv_it + j) % kStages) ? dv1 : dv0;
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
      auto wait_k = [&](int j) {
        const int it = kv_it + j;
        return wwait(kBarKFull + it % kStages, (it / kStages) & 1);
      };
      // PV_t(j).  With want_k the next K tile is checked while the second half
      // of P is still being written, so that PV's second half and S_t(j+1)
      // issue back to back once P is complete.
      auto issue_pv = [&](int t, int j, bool want_k) -> bool {
        if (!wwait(kBarPHalf + t, p_it[t] & 1)) return false;
        tc_fence_after();
        issue_pv_half(t, j, 0);
        if (want_k && !wait_k(j + 1)) return false;
        if (!wwait(kBarPFull + t, p_it[t] & 1)) return false;
        tc_fence_after();
        issue_pv_half(t, j, BN / 32);
        if (leader) mma_commit(bar(kBarODone + t));
        __syncwarp();
        ++p_it[t];
        return true;
      };

      ok = wait_k(0);
#pragma unroll
      for (int t = 0; t < kQTiles; ++t) {
        if (!ok || g.n[t] == 0) continue;
        ok = wwait(kBarQFull + t, q_it[t] & 1);
        if (!ok) continue;
        tc_fence_after();
        issue_s(t, 0);
      }
      if (ok) commit(kBarKEmpty + kv_it % kStages);
      for (int j = 0; j < nmax && ok; ++j) {
        const int it = kv_it + j;
        const int st = it % kStages;
        if (last_fix && j == nmax - 1)
          ok = wwait(kBarVFixed, tail_it & 1);
        else
          ok = wwait(kBarVFull + st, (it / kStages) & 1);
        bool have_k = false;
#pragma unroll
        for (int t = 0; t < kQTiles; ++t) {
          if (!ok || j >= g.n[t]) continue;
          const bool more = j + 1 < g.n[t];
          ok = issue_pv(t, j, more && !have_k);
          if (!ok) continue;
          have_k = have_k || more;
          if (more) {
            tc_fence_after();
            issue_s(t, j + 1);
          }
        }
        if (!ok) break;
        commit(kBarVEmpty + st);
        if (j + 1 < nmax) commit(kBarKEmpty + (it + 1) % kStages);
      }
      kv_it += nmax;
      tail_it += last_fix;
#pragma unroll
      for (int t = 0; t < kQTiles; ++t) q_it[t] += g.n[t] > 0;
    }
    if (!ok) {
      // Let every MMA already issued finish before TMEM is released.
      if (leader) mma_commit(bar(kBarDrain));
      __syncwarp();
      mbar_wait_bounded(bar(kBarDrain), 0, limit_ns);
    }
  } else if (warp < 8) {
    // ------------------------------------------------------------- softmax --
    regs_increase<kRegsSoftmax>();
    const int t = warp >> 2;                         // Q tile of this warpgroup
    const int r = threadIdx.x & 127;                 // row in tile = TMEM lane
    const uint32_t lane_addr = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + lane_addr + kColS + 128 * t;
    const uint32_t tO = tmem + lane_addr + kColO + 128 * t;
    const float c = p.scale_log2;
    const int box_shift = kPaged ? min(p.page_shift, 7) : 7;   // log2(rows per page box)
    int kv_it = 0, s_it = 0;
    bool ok = true;
    for (int k = 0; ok; ++k) {
      const int item = k == 0 ? blockIdx.x : read_item(k - 1);
      if (item == -2) ok = false;
      if (item < 0) break;
      const Geometry g = item_geometry(p, item);
      const int n = g.n[t];
      const int row = g.q0 + t * BM + r;             // query row
      const int limit = p.causal ? min(row + g.off, g.kv_len - 1) : g.kv_len - 1;
      float m_ref = -INFINITY, l = 0.f;
      // tcgen05.ld/st are warp-collective: every branch around them is warp-uniform.
      for (int j = 0; j < n; ++j) {
        ok = __all_sync(0xffffffffu, wait(kBarSFull + t, s_it & 1));
        if (!ok) break;
        ++s_it;
        uint32_t bad_keys[4] = {0u, 0u, 0u, 0u};      // keys of pages outside the pool
        if (kPaged) {
          // Keys of pages outside the pool are left out (their K rows were
          // never loaded).  The loader wrote this tile's mask before its K load.
          const int it = kv_it + j;
          uint32_t w = mask_slot[it % kMaskSlots];
          if ((w >> 8) != static_cast<uint32_t>(it & 0xFFFFFF)) {
            const uint64_t t0 = globaltimer_ns();
            while ((w >> 8) != static_cast<uint32_t>(it & 0xFFFFFF)) {
              if (*abort_flag || globaltimer_ns() - t0 > limit_ns) {
                fail();
                break;
              }
              w = mask_slot[it % kMaskSlots];
            }
          }
          if (!__all_sync(0xffffffffu, !*abort_flag)) {   // the mask wait gave up
            ok = false;
            break;
          }
          const uint32_t bad_boxes = w & 0xFFu;           // same on every lane
          if (bad_boxes) {
            // A box is 16 keys (16-token pages: two boxes per word) or a
            // multiple of 32 keys (one box covers whole words).
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              if (box_shift == 4)
                bad_keys[q] = (((bad_boxes >> (2 * q)) & 1u) ? 0x0000FFFFu : 0u) |
                              (((bad_boxes >> (2 * q + 1)) & 1u) ? 0xFFFF0000u : 0u);
              else
                bad_keys[q] = ((bad_boxes >> ((32 * q) >> box_shift)) & 1u) ? 0xFFFFFFFFu : 0u;
            }
          }
        }
        tc_fence_after();
        uint32_t s[128];
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
          uint32_t (&sub)[32] = *reinterpret_cast<uint32_t(*)[32]>(&s[32 * ch]);
          tmem_ld32(tS + 32 * ch, sub);
        }
        tmem_wait_ld();
        const int k0 = j * BN;
        // Diagonal or tail tile, or keys of a bad page: one masking pass over
        // a bit per key (bit b of word q = key k0 + 32 q + b is hidden).
        const bool masked = k0 + BN - 1 > limit ||
                            (kPaged && (bad_keys[0] | bad_keys[1] | bad_keys[2] | bad_keys[3]));
        if (masked) {
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int first_hidden = limit + 1 - (k0 + 32 * q);     // keys >= this are hidden
            uint32_t hide = first_hidden <= 0 ? 0xFFFFFFFFu
                          : first_hidden >= 32 ? 0u : (0xFFFFFFFFu << first_hidden);
            if (kPaged) hide |= bad_keys[q];
#pragma unroll
            for (int b = 0; b < 32; ++b)
              if ((hide >> b) & 1u) s[32 * q + b] = __float_as_uint(-INFINITY);
          }
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
        const uint64_t c2 = f2(c, c);
        uint64_t acc[4];
        auto exp_half = [&](int ch, float neg_m, uint32_t (&pk)[32]) {
          const uint64_t nm2 = f2(neg_m, neg_m);
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const int e = 64 * ch + 2 * i;
            const uint64_t x2 = fma2(f2(__uint_as_float(s[e]), __uint_as_float(s[e + 1])), c2, nm2);
            float x0, x1;
            unf2(x2, x0, x1);
            const float p0 = ex2(x0);
            const float p1 = ex2(x1);
            acc[i & 3] = add2(acc[i & 3], f2(p0, p1));
            pk[i] = pack_bf16x2(p0, p1);
          }
        };
#pragma unroll
        for (int a = 0; a < 4; ++a) acc[a] = f2(0.f, 0.f);
        uint32_t pk[32];
        const float m_tile = mx * c;                  // running max in log2 units
        float alpha = 1.f;
        bool rescale = false;
        if (m_tile > m_ref + kRescaleThreshold || (m_ref == -INFINITY && m_tile != -INFINITY)) {
          alpha = ex2(m_ref - m_tile);               // m_ref = -inf -> 0
          m_ref = m_tile;
          rescale = true;
        }
        const float neg_m = (m_ref == -INFINITY) ? 0.f : -m_ref;
        exp_half(0, neg_m, pk);
        if (__any_sync(0xffffffffu, rescale) && j > 0) {
          // O must be rescaled before PV(j) may start, i.e. before any P is
          // handed over; PV(j-1) has completed (S(j) was issued after it).
          // alpha = 1 in rows that keep m.
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
        tmem_st32(tS, pk);
        tmem_wait_st();                              // first half of P: PV(j) may start
        tc_fence_before();
        mbar_arrive(bar(kBarPHalf + t));
        exp_half(1, neg_m, pk);
        tmem_st32(tS + 32, pk);
        float s0, s1;
        unf2(add2(add2(acc[0], acc[1]), add2(acc[2], acc[3])), s0, s1);
        l = l * alpha + (s0 + s1);
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(bar(kBarPFull + t));
      }
      if (!ok) break;
      // Epilogue: O / l -> bf16 -> global (rows past q_len are not stored).
      // PV_t of this item's last tile is the (s_it - 1)-th PV of this tile.
      if (n > 0) {
        ok = __all_sync(0xffffffffu, wait(kBarODone + t, (s_it - 1) & 1));
        if (!ok) break;
        tc_fence_after();
      }
      const bool store = row < p.q_len;
      __nv_bfloat16* out = static_cast<__nv_bfloat16*>(p.O) +
                           (((size_t)g.b * p.H + g.h) * p.q_len + (store ? row : 0)) * D;
      const float inv = (n > 0 && l > 0.f) ? 1.f / l : 0.f;
#pragma unroll
      for (int ch = 0; ch < 4; ++ch) {
        uint32_t o[32];
        if (n > 0) {
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
      kv_it += g.nmax;
    }
    // No tensor-memory access of this warp may still be in flight at dealloc.
    tmem_wait_ld();
    tmem_wait_st();
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

// Dynamic shared memory is a per-device function attribute; host threads may
// launch concurrently, so the once-per-device record is kept under a lock.
template <bool kPaged, bool kFp8QK>
cudaError_t set_smem_attr() {
  static bool done[64] = {};
  static std::mutex mu;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(mu);
  if (dev >= 0 && dev < 64 && done[dev]) return cudaSuccess;
  // The in-kernel register split assumes this exact launch allocation (the
  // build checks it too).
  cudaFuncAttributes fa;
  e = cudaFuncGetAttributes(&fa, prefill_kernel<kPaged, kFp8QK>);
  if (e != cudaSuccess) return e;
  if (fa.numRegs != kLaunchRegs) return cudaErrorNotSupported;
  e = cudaFuncSetAttribute(prefill_kernel<kPaged, kFp8QK>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           kSmemBytes);
  if (e == cudaSuccess && dev >= 0 && dev < 64) done[dev] = true;
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
  // One CTA per work item; running CTAs claim the items of CTAs that have not
  // started (so at most one CTA per SM ever runs, and the rest never launch).
  const long long m_blocks = (p.q_len + BM * kQTiles - 1) / (BM * kQTiles);
  const long long ctas = m_blocks * p.B * p.H;
  if (ctas > 0x7fffffffLL) return cudaErrorNotSupported;
  dim3 grid((unsigned)ctas);
  // Heads scheduled together: as many as keep about 64 MB of K/V live in L2
  // (query heads sharing a kv head count once; measured ahead of 16 and 32 MB).
  PrefillParams q = p;
  {
    const long long kv_len = p.paged ? p.max_seq_len : p.kv_len;
    const long long kv_bytes = 2LL * kv_len * D * 2;              // K and V of one kv head
    const int group_q = p.H / p.H_kv;
    long long hg = (64LL << 20) / (kv_bytes > 0 ? kv_bytes : 1) * group_q;
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
