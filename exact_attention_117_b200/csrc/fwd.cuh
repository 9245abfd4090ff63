// fwd.cuh -- forward attention kernel for sm_100a.
//
// Algorithm (page "从零实现 FlashAttention-2：分块在线 Softmax", sections
// 在线 softmax：重缩放恒等式 and 从 FlashAttention-1 到 FlashAttention-2; page
// "FlashAttention 为什么能节省显存并提速,是否改变注意力结果?", section
// 难点在于分块后softmax如何归一): Q tiles stay on chip while 128-key K/V
// tiles stream past; per key tile the running row max m and sum l are updated,
// the output accumulator is rescaled by exp(m_old - m_new), and O += P V
// accumulates; O / l and the row logsumexp are written once at the end.  No
// N x N tensor ever reaches global memory.
//
// A work item is TWO consecutive 128-row Q tiles of one (batch, head) (and,
// for the split-KV forward, one range of key tiles); the CTA runs the two
// tiles ping-pong: while the softmax warps of one tile work on its scores, the
// tensor core computes P V and the next S = Q K^T of the other tile.
//
// The kernel is persistent: about one CTA per SM, each taking items until
// none are left (the first from blockIdx.x, the rest from a per-launch work
// counter, longest items first).  The K/V ring and every barrier phase run on
// across items, so the next item's Q and first K/V tiles load, and its first
// scores are computed, while the previous item's last tiles and epilogue are
// still in flight; the epilogue stores O through two small staging boxes per
// softmax warp (TMA stores), so it holds no shared memory the next item needs.
//
// Warp roles (384 threads):
//   warp 0      : TMA producer (an item's two Q tiles, then its K_j / V_j) and
//                 scheduler: once an item's loads are issued it takes the next
//                 item from the counter and publishes it in a two-slot ring
//                 that the other roles read (an item is claimed only when this
//                 CTA is about to load it, so the counter keeps the balance;
//                 claiming it as the previous item's loads start was measured
//                 7 % slower on B=2 H=16 N=4096)
//   warp 1      : TMEM allocator and tcgen05.mma issuer
//   warps 2-3   : idle
//   warps 4-7   : softmax of Q tile 0, one thread per query row
//   warps 8-11  : softmax of Q tile 1
// (TMEM lane = row, so a row's max and sum stay inside one thread.)
//
// TMEM columns: S0 [0,128), S1 [128,256), O0 [256,256+D), O1 [256+D,256+2D).
// The bf16 probabilities P_t are written over the first 64 columns of S_t and
// fed to the P V product as the TMEM A operand.  tcgen05.mma ops from one
// thread run in issue order, so S_t(j+1) may be issued right after the P V
// product that reads P_t(j) from the same columns.  A tcgen05.commit arrives
// only when every earlier MMA of the issuing thread is complete, so when a
// softmax warp sees S_t(j) ready, P_t(j-1) V is done and O_t is current.
//
// Rescaling (page 2, section 提示: the factor is exactly 1 when the max is
// unchanged): a row keeps its running max until a tile raises it by more than
// 8 (base-2 units); until then the new probabilities are taken against the
// old max (they are at most 2^8) and O needs no correction.  O and l always
// refer to the same max, so O / l and m + log2 l are unchanged in exact
// arithmetic.  The rescale of O in TMEM is done only when some row of the
// warp moved its max.
//
// Causal masking (page 2, section 提示): key tiles wholly above a Q tile's
// diagonal are never computed for it; the diagonal tile masks key > query.
// All exponentials are base 2 with scale*log2(e) folded in; the stored LSE is
// converted back to natural log.
#pragma once

#include <cuda_bf16.h>

#include "common.cuh"

namespace fa {

template <int D>
struct FwdLayout {
  static constexpr int kBM = 128;                    // query rows per Q tile
  static constexpr int kBN = 128;                    // keys per K/V tile
  static constexpr int kStages = (D == 64) ? 4 : 2;  // K and V ring depth
  static constexpr int kTile = kBM * D * 2;          // bytes of a Q, K or V tile
  static constexpr int kOffQ0 = 0;
  static constexpr int kOffQ1 = kTile;
  static constexpr int kOffK = 2 * kTile;
  static constexpr int kOffV = kOffK + kStages * kTile;
  // O staging for the TMA stores of the epilogue: per softmax warp two 32 x 32
  // bf16 boxes (64-byte rows, 64-byte swizzle), used alternately
  static constexpr int kStageBytes = 32 * 32 * 2;
  static constexpr int kOffStage = kOffV + kStages * kTile;
  static constexpr int kOffBar = kOffStage + 8 * 2 * kStageBytes;
  static constexpr int kBarArea = 512;
  static constexpr int kBytes = kOffBar + kBarArea;
  static constexpr int kSmemAlloc = kBytes + 1024;  // slack to align the base to 1 KiB
  // barrier indices
  static constexpr int kQFull = 0;
  static constexpr int kQEmpty = 1;
  static constexpr int kKFull = 2;
  static constexpr int kKEmpty = kKFull + kStages;
  static constexpr int kVFull = kKEmpty + kStages;
  static constexpr int kVEmpty = kVFull + kStages;
  // S ready / P ready, one barrier per score buffer (two, or three at d = 64)
  static constexpr int kSFull = kVEmpty + kStages;  // [3]
  static constexpr int kPFull = kSFull + 3;         // [3]
  static constexpr int kOFinal = kPFull + 3;        // [2]
  static constexpr int kPvDone = kOFinal + 2;       // [2] one phase per P V of the tile
  static constexpr int kItemFull = kPvDone + 2;     // [2]
  static constexpr int kItemEmpty = kItemFull + 2;  // [2]
  static constexpr int kDrain = kItemEmpty + 2;
  static constexpr int kNumBars = kDrain + 1;
  static constexpr int kOffSlot = kOffBar + 8 * kNumBars;  // TMEM base address
  static constexpr int kOffAbort = kOffSlot + 4;
  static constexpr int kOffItems = kOffAbort + 4;  // [2] item ring
  static_assert(kOffItems + 8 <= kOffBar + kBarArea, "barrier area too small");
  static_assert(kSmemAlloc <= 232448, "shared memory budget");
  static constexpr uint32_t kTmemCols = 512;
  // d = 128: S0, S1, O0, O1 fill the 512 columns.  d = 64: three score buffers
  // shared by the two tiles, then O0, O1 (see s_ref below).
  static constexpr bool kThreeS = (D == 64);
  static constexpr uint32_t kColS0 = 0, kColS1 = 128;
  static constexpr uint32_t kColO0 = kThreeS ? 384 : 256, kColO1 = kColO0 + D;
  static constexpr float kRescaleThreshold = 8.0f;    // base-2 units
  static constexpr float kSpecRedoThreshold = 20.0f;  // base-2 units, speculative tiles
  static constexpr uint32_t kLaunchRegs = 168;      // 65536 / 384, rounded down to 8
  static constexpr uint32_t kRegsOther = 80;
  static constexpr uint32_t kRegsSoftmax = 200;
  static_assert(128 * kRegsOther + 256 * kRegsSoftmax <= 384 * kLaunchRegs, "register split");
  // arrivals that free an item ring slot: MMA warp, 8 softmax warps
  static constexpr uint32_t kItemReaders = 9;
};

// One work item: Q tiles qt0 and qt1 of slice bh, key tiles [kb, kb + n1).
struct FwdItem {
  int bh, qt0, qt1, kb, n0, n1, split;
  bool single;  // odd tile count: only qt1 (== qt0) is real, tile 0 idles
};

// Item order: heads in groups of head_group; within a group the pairs with
// the most key tiles come first, every head of the group at each pair; the
// splits of one (head, pair) are consecutive.  The CTAs busy at any time then
// read the K/V of a bounded set of heads, which stays in L2.
template <bool kCausal, bool kSplit>
__device__ __forceinline__ FwdItem fwd_item(int item, int n_kv_all, int bh_count, int head_group,
                                            int num_splits) {
  FwdItem w;
  const int n_pairs = (n_kv_all + 1) / 2;
  w.split = kSplit ? item % num_splits : 0;
  const int lin = kSplit ? item / num_splits : item;
  const int grp = lin / (head_group * n_pairs);
  const int g_base = grp * head_group;
  const int g_size = min(head_group, bh_count - g_base);
  const int g_off = lin - grp * head_group * n_pairs;
  const int pair = n_pairs - 1 - g_off / g_size;
  w.bh = g_base + g_off % g_size;
  w.single = 2 * pair + 1 >= n_kv_all;
  w.qt0 = 2 * pair;
  w.qt1 = w.single ? 2 * pair : 2 * pair + 1;
  int kb = 0, ke = n_kv_all;
  if (kSplit) {
    const int chunk = (n_kv_all + num_splits - 1) / num_splits;
    kb = w.split * chunk;
    ke = min(kb + chunk, n_kv_all);
  }
  const int end0 = kCausal ? min(w.qt0 + 1, n_kv_all) : n_kv_all;
  const int end1 = kCausal ? min(w.qt1 + 1, n_kv_all) : n_kv_all;
  w.kb = kb;
  w.n0 = w.single ? 0 : max(0, min(ke, end0) - kb);
  w.n1 = max(0, min(ke, end1) - kb);  // n1 >= n0; a split may have 0
  return w;
}

// Where the score tile S_t(j) of an item lives (n0 key tiles for Q tile 0):
// its TMEM column, the index of its S-ready / P-ready barriers and the parity
// of the phase that stands for it.  With two buffers, tile t always uses
// buffer t and the phases count tile t's key steps (t_steps of them before
// this one).  With three (d = 64), the score tiles take the buffers in turn
// in the order the MMA warp issues them -- S_0(0), S_1(0), then per key step
// S_0(j+1), S_1(j+1) -- so that a tile's next scores are computed into the
// third buffer while its softmax still reads the current ones; s_base counts
// the score tiles of earlier items.  A buffer is reused only after the P V
// that reads it, so its barriers never run two phases ahead of a waiter.
struct SRef {
  uint32_t col;
  int buf;
  uint32_t parity;
};
template <int D>
__device__ __forceinline__ SRef s_ref(int t, int j, int n0, int s_base, int t_steps) {
  using L = FwdLayout<D>;
  if (!L::kThreeS)
    return {t ? L::kColS1 : L::kColS0, t, static_cast<uint32_t>(t_steps & 1)};
  // the issue index of S_t(j) in this item: tile 0 has n0 tiles, tile 1 n1 =
  // n0 or n0 + 1 (or n1 alone when tile 0 idles, n0 = 0)
  const int k = s_base + ((t == 0) ? 2 * j : (j < n0 ? 2 * j + 1 : n0 + j));
  return {static_cast<uint32_t>(k % 3) * 128, k % 3, static_cast<uint32_t>((k / 3) & 1)};
}

// kSplit: an item covers only the key tiles of its split (a contiguous range
// of ceil(n_kv / num_splits) tiles) and writes, instead of O and LSE, fp32
// partial results: O_s = u_s / l_s in the tile layout [D/4 column groups][128
// rows][4] of part_o, and LSE_s = m_s + log2 l_s (base 2) in part_lse; a split
// that sees no key of a row writes O_s = 0, LSE_s = -inf.
// splitkv_combine_kernel merges the splits.
template <int D, bool kCausal, bool kSplit>
__global__ void __launch_bounds__(384, 1)
    fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
               const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
               float* __restrict__ lse_out, int n, int bh_count, float scale_log2,
               uint64_t limit_ns, int num_splits, float* __restrict__ part_o,
               float* __restrict__ part_lse, int head_group, int n_items, uint32_t sched_slot) {
  using L = FwdLayout<D>;
  constexpr int S = L::kStages;
  constexpr int kDBlk = D / 64;  // 128-byte swizzle blocks per tile row

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
  const uint32_t sb = smem_u32(smem);
  auto bar = [&](int i) -> uint32_t { return sb + L::kOffBar + 8u * static_cast<uint32_t>(i); };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kOffAbort);
  volatile int* item_ring = reinterpret_cast<volatile int*>(smem + L::kOffItems);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kOffSlot);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int n_kv_all = (n + L::kBN - 1) / L::kBN;  // also the number of Q tiles (Nq = Nk)
  const unsigned int err_fwd = kErrFwd;

  if (threadIdx.x == 0) {
    for (int b = 0; b < L::kNumBars; ++b) {
      uint32_t cnt = 1;
      if (b >= L::kPFull && b < L::kPFull + 3) cnt = 4;
      if (b == L::kItemEmpty || b == L::kItemEmpty + 1) cnt = L::kItemReaders;
      mbar_init(bar(b), cnt);
    }
    *abort_flag = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), L::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // Item k of this CTA from the ring (warp-uniform); false if the wait gave
  // up.  Every reader arrives once per item on the slot's empty barrier
  // (lane 0 of each reading warp).
  auto read_item = [&](int k, int& item, unsigned int err) -> bool {
    if (!wait_bounded_warp(bar(L::kItemFull + (k & 1)), (k >> 1) & 1, limit_ns, abort_flag, err))
      return false;
    item = item_ring[k & 1];
    __syncwarp();
    if (lane == 0) mbar_arrive(bar(L::kItemEmpty + (k & 1)));
    return true;
  };

  // Registers: the block launches with 168 per thread (384 x 168 = 64512).
  // Load / MMA / idle warps drop to 80, the two softmax warp groups rise
  // to 200: 128 x 80 + 256 x 200 = 61440 <= 64512.
  if (warp < 4) {
    setmaxnreg_dec<L::kRegsOther>();
    if (warp == 0) {
      // --------------------------------------------------- producer, scheduler
      const uint32_t err = err_fwd | kErrRoleLoad;
      if (lane == 0) {
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
      }
      int g_kv = 0;   // K/V tiles issued so far (ring position)
      int q_cnt = 0;  // items whose Q tiles were loaded
      bool q_pending = false;
      int nk = 0, nv = 0;  // K and V tiles issued
      // publishes item k (or -1: no more work) in ring slot k & 1 once every
      // reader has taken item k - 2 from it
      auto publish = [&](int k, int item) -> bool {
        bool ok = true;
        if (lane == 0) {
          ok = wait_bounded(bar(L::kItemEmpty + (k & 1)), ((k >> 1) & 1) ^ 1, limit_ns, abort_flag,
                            err);
          if (ok) {
            item_ring[k & 1] = item;
            mbar_arrive(bar(L::kItemFull + (k & 1)));  // release: readers acquire the slot
          }
        }
        return __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      };
      int item = static_cast<int>(blockIdx.x);
      for (int k = 0; publish(k, item); ++k) {
        if (item < 0) break;
        const FwdItem w = fwd_item<kCausal, kSplit>(item, n_kv_all, bh_count, head_group, num_splits);
        if (lane == 0 && w.n1 > 0) {
          bool ok = true;
          // the Q buffers are free once the previous item's last S MMA is done
          if (q_cnt > 0)
            ok = wait_bounded(bar(L::kQEmpty), (q_cnt - 1) & 1, limit_ns, abort_flag, err);
          ok = ok && dbg_check(w.qt0 >= 0 && w.qt1 * L::kBM < n && w.bh >= 0 && w.bh < bh_count &&
                                   w.kb >= 0 && w.kb + w.n1 <= n_kv_all,
                               err, abort_flag);
          if (ok) {
            mbar_arrive_expect_tx(bar(L::kQFull), (w.single ? 1 : 2) * L::kTile);
            for (int db = 0; db < kDBlk; ++db) {
              if (!w.single)
                tma_load_3d(sb + L::kOffQ0 + db * 16384, &tm_q, bar(L::kQFull), db * 64,
                            w.qt0 * L::kBM, w.bh);
              tma_load_3d(sb + L::kOffQ1 + db * 16384, &tm_q, bar(L::kQFull), db * 64,
                          w.qt1 * L::kBM, w.bh);
            }
            q_pending = true;
          }
          for (int jj = 0; ok && jj < w.n1; ++jj) {
            const int gi = g_kv + jj;
            const int j = w.kb + jj;  // key tile
            const int s = gi % S;
            const uint32_t ph = (gi / S) & 1;
            if (!dbg_check(j * L::kBN < n && L::kOffV + (s + 1) * L::kTile <= L::kOffBar, err,
                           abort_flag) ||
                !wait_bounded(bar(L::kKEmpty + s), ph ^ 1, limit_ns, abort_flag, err)) {
              ok = false;
              break;
            }
            mbar_arrive_expect_tx(bar(L::kKFull + s), L::kTile);
            for (int db = 0; db < kDBlk; ++db)
              tma_load_3d(sb + L::kOffK + s * L::kTile + db * 16384, &tm_k, bar(L::kKFull + s),
                          db * 64, j * L::kBN, w.bh);
            ++nk;
            if (!wait_bounded(bar(L::kVEmpty + s), ph ^ 1, limit_ns, abort_flag, err)) {
              ok = false;
              break;
            }
            mbar_arrive_expect_tx(bar(L::kVFull + s), L::kTile);
            for (int db = 0; db < kDBlk; ++db)
              tma_load_3d(sb + L::kOffV + s * L::kTile + db * 16384, &tm_v, bar(L::kVFull + s),
                          db * 64, j * L::kBN, w.bh);
            ++nv;
          }
          if (!ok) item = -2;  // leave the item loop (after the drain below)
        }
        if (__shfl_sync(0xffffffffu, item, 0) == -2) break;
        if (w.n1 > 0) {
          ++q_cnt;
          g_kv += w.n1;
        }
        // claim the next item now that this one's loads are all issued
        unsigned int f = 0;
        if (lane == 0) f = atomicAdd(&g_sched_next[sched_slot], 1u);
        f = __shfl_sync(0xffffffffu, f, 0);
        item = f >= static_cast<unsigned int>(n_items) - gridDim.x ? -1
                                                                    : static_cast<int>(gridDim.x + f);
      }
      if (lane == 0 && *abort_flag && q_pending) {
        // let every copy already issued land before shared memory is released
        drain_wait(bar(L::kQFull), (q_cnt - 1) & 1, limit_ns);
        for (int j = (nk > S ? nk - S : 0); j < nk; ++j)
          drain_wait(bar(L::kKFull + j % S), (j / S) & 1, limit_ns);
        for (int j = (nv > S ? nv - S : 0); j < nv; ++j)
          drain_wait(bar(L::kVFull + j % S), (j / S) & 1, limit_ns);
      }
    } else if (warp == 1) {
      // ------------------------------------------------------------ MMA issuer
      // the whole warp runs this loop; the MMA and commit wrappers elect one lane
      constexpr uint32_t id_s = idesc_bf16_f32(128, 128, false, false);
      constexpr uint32_t id_o = idesc_bf16_f32(128, D, false, true);
      const uint32_t err = err_fwd | kErrRoleMma;
      int s_base = 0;  // score tiles issued by earlier items
      // The two issue loops below are unrolled by 2, not fully: they are
      // expanded at several places of this loop, and the smaller code leaves
      // more of the instruction cache to the softmax warps (B200, against
      // full unrolling: B=64 H=16 N=1024 causal +13 %, B=2 H=16 N=4096 +1.4 %,
      // B=1 H=32 N=16384 -1.4 %; not unrolled at all: B=2 H=16 N=4096 -7 %).
      // S_t(j) = Q_t K^T, K from ring position gi
      auto issue_s = [&](int t, int gi, int j, int n0) {
        const uint32_t qa = sb + (t ? L::kOffQ1 : L::kOffQ0);
        const uint32_t ka = sb + L::kOffK + (gi % S) * L::kTile;
        const SRef sr = s_ref<D>(t, j, n0, s_base, 0);
        const uint32_t d_tmem = tmem + sr.col;
#pragma unroll 2
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
          mma_bf16_ss(d_tmem, sw128_desc(qa + off, 16, 1024), sw128_desc(ka + off, 16, 1024), id_s,
                      kk > 0 ? 1u : 0u);
        }
        tc_commit(bar(L::kSFull + sr.buf));
      };
      // O_t (+)= P_t(j) V, P_t(j) from TMEM over S_t(j)
      auto issue_pv = [&](int t, int gi, bool first, int j, int n0) {
        const uint32_t va = sb + L::kOffV + (gi % S) * L::kTile;
        const uint32_t d_tmem = tmem + (t ? L::kColO1 : L::kColO0);
        const uint32_t a_tmem = tmem + s_ref<D>(t, j, n0, s_base, 0).col;
#pragma unroll 2
        for (int kk = 0; kk < L::kBN / 16; ++kk)
          mma_bf16_ts(d_tmem, a_tmem + kk * 8, sw128_desc(va + kk * 2048, 16384, 1024), id_o,
                      (!first || kk > 0) ? 1u : 0u);
      };
      int g_kv = 0, q_cnt = 0, p0 = 0, p1 = 0;
      bool ok = true;
      for (int k = 0; ok; ++k) {
        int item;
        if (!read_item(k, item, err)) break;
        if (item < 0) break;
        const FwdItem w = fwd_item<kCausal, kSplit>(item, n_kv_all, bh_count, head_group, num_splits);
        const int n0 = w.n0, n1 = w.n1;
        if (n1 == 0) continue;
        ok = dbg_check(tmem_range_ok(tmem + L::kColO1, tmem, D, L::kTmemCols) &&
                           tmem_range_ok(tmem + L::kColS1, tmem, 128, L::kTmemCols),
                       err, abort_flag) &&
             wait_bounded_warp(bar(L::kQFull), q_cnt & 1, limit_ns, abort_flag, err) &&
             wait_bounded_warp(bar(L::kKFull + g_kv % S), (g_kv / S) & 1, limit_ns, abort_flag, err);
        ++q_cnt;
        if (!ok) break;
        tc_fence_after();
        if (n0 > 0) issue_s(0, g_kv, 0, n0);
        issue_s(1, g_kv, 0, n0);
        tc_commit(bar(L::kKEmpty + g_kv % S));
        if (n1 == 1) tc_commit(bar(L::kQEmpty));  // the item's last S reads of Q are issued
        for (int jj = 0; jj < n1; ++jj) {
          const int gi = g_kv + jj;
          const int s = gi % S;
          if (!wait_bounded_warp(bar(L::kVFull + s), (gi / S) & 1, limit_ns, abort_flag, err)) {
            ok = false;
            break;
          }
          const bool next = jj + 1 < n1;
          const int s1 = (gi + 1) % S;
          // three buffers: tile 0's next scores go into the free buffer before
          // its current P V; two buffers: after it, into the same buffer
          if (L::kThreeS && next) {
            if (!wait_bounded_warp(bar(L::kKFull + s1), ((gi + 1) / S) & 1, limit_ns, abort_flag,
                                   err)) {
              ok = false;
              break;
            }
            tc_fence_after();
            if (jj + 1 < n0) issue_s(0, gi + 1, jj + 1, n0);
          }
          if (jj < n0) {
            const SRef pr = s_ref<D>(0, jj, n0, s_base, p0);
            if (!wait_bounded_warp(bar(L::kPFull + pr.buf), pr.parity, limit_ns, abort_flag, err)) {
              ok = false;
              break;
            }
            ++p0;
            tc_fence_after();
            issue_pv(0, gi, jj == 0, jj, n0);
            tc_commit(bar(L::kPvDone + 0));
            if (jj == n0 - 1) tc_commit(bar(L::kOFinal + 0));
          }
          if (next) {
            if (!L::kThreeS) {
              if (!wait_bounded_warp(bar(L::kKFull + s1), ((gi + 1) / S) & 1, limit_ns, abort_flag,
                                     err)) {
                ok = false;
                break;
              }
              tc_fence_after();
              if (jj + 1 < n0) issue_s(0, gi + 1, jj + 1, n0);
            } else {
              // tile 1's next scores into the buffer tile 0's P V has just
              // been issued from
              issue_s(1, gi + 1, jj + 1, n0);
              tc_commit(bar(L::kKEmpty + s1));
              if (jj + 2 == n1) tc_commit(bar(L::kQEmpty));  // last S reads of Q issued
            }
          }
          const SRef pr1 = s_ref<D>(1, jj, n0, s_base, p1);
          if (!wait_bounded_warp(bar(L::kPFull + pr1.buf), pr1.parity, limit_ns, abort_flag, err)) {
            ok = false;
            break;
          }
          ++p1;
          tc_fence_after();
          issue_pv(1, gi, jj == 0, jj, n0);
          tc_commit(bar(L::kPvDone + 1));
          if (jj == n1 - 1) tc_commit(bar(L::kOFinal + 1));
          tc_commit(bar(L::kVEmpty + s));
          if (next && !L::kThreeS) {
            issue_s(1, gi + 1, jj + 1, n0);
            tc_commit(bar(L::kKEmpty + s1));
            if (jj + 2 == n1) tc_commit(bar(L::kQEmpty));  // last S reads of Q issued
          }
        }
        s_base += n0 + n1;
        g_kv += n1;
      }
      // every MMA issued above must finish before TMEM / smem are released
      tc_commit(bar(L::kDrain));
      drain_wait(bar(L::kDrain), 0, limit_ns);
      __syncwarp();
    }
  } else {
    setmaxnreg_inc<L::kRegsSoftmax>();
    // ------------------------------------------------- softmax / epilogue
    const int t = (warp >= 8) ? 1 : 0;         // which Q tile
    const int r = threadIdx.x - 128 - 128 * t;  // row inside the tile == TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t o_addr = tmem + lane_off + (t ? L::kColO1 : L::kColO0);
    const uint32_t err = err_fwd | kErrRoleSoftmax;
    const bool neg_scale = scale_log2 < 0.f;
    const uint32_t masked_bits = __float_as_uint(neg_scale ? INFINITY : -INFINITY);
    int s_cnt = 0, of_cnt = 0;  // S tiles and final O of this tile seen so far
    int s_base = 0;             // score tiles of earlier items
    // Before a rescale of O_t at key step jj > 0: O_t holds the tiles before
    // jj once their P V has finished.  With two buffers the S_t(jj) seen ready
    // was issued after that P V, so it has; with three it was issued before it.
    auto o_current = [&]() -> bool {
      if (!L::kThreeS) return true;
      const bool got =
          wait_bounded_warp(bar(L::kPvDone + t), (s_cnt - 2) & 1, limit_ns, abort_flag, err);
      tc_fence_after();
      return got;
    };
    int st_cnt = 0;             // O boxes this warp has stored (staging buffer st_cnt & 1)
    const int sw = warp - 4;    // softmax warp 0..7: its staging buffers
    bool ok = true;
    for (int k = 0; ok; ++k) {
      int item;
      if (!read_item(k, item, err) || item < 0) break;
      const FwdItem w = fwd_item<kCausal, kSplit>(item, n_kv_all, bh_count, head_group, num_splits);
      const int qt = t ? w.qt1 : w.qt0;
      const int n_t = t ? w.n1 : w.n0;
      const bool active = t == 1 || !w.single;  // this tile stands for a real Q tile
      float m_run = -INFINITY;  // running (possibly stale) max of scale*log2(e)*s
      float l_run = 0.f;        // running sum of 2^(x - m_run)
      if (!dbg_check(tmem_range_ok(tmem + lane_off + L::kColS0, tmem, L::kThreeS ? 384 : 256,
                                   L::kTmemCols) &&
                         tmem_range_ok(o_addr, tmem, D, L::kTmemCols) && qt < n_kv_all &&
                         w.bh < bh_count && w.split < num_splits,
                     err, abort_flag))
        break;
      for (int jj = 0; jj < n_t; ++jj) {
        const int j = w.kb + jj;  // key tile
        const SRef sr = s_ref<D>(t, jj, w.n0, s_base, s_cnt);
        if (!wait_bounded_warp(bar(L::kSFull + sr.buf), sr.parity, limit_ns, abort_flag, err)) {
          ok = false;
          break;
        }
        ++s_cnt;
        tc_fence_after();
        const uint32_t s_addr = tmem + lane_off + sr.col;
        uint32_t u[128];  // raw fp32 scores of this row
        int lim = L::kBN;
        if (kCausal && j == qt) lim = r + 1;
        const int rem = n - j * L::kBN;
        if (rem < lim) lim = rem;
        // From the second key tile on (positive scale) the
        // exponentials are taken against the running max right away, while the
        // tile's max is found alongside, and the second half of the row loads
        // while the first half is exponentiated: the max is off the critical
        // path.  A row's probabilities then reach 2^(tile max - running max);
        // up to 2^20 that is harmless (bf16 P and the fp32 sums have the range,
        // and O and l stay relative to the same max), so only a jump beyond
        // that -- never seen with these inputs -- redoes the tile.
        if (jj > 0 && !neg_scale && !__any_sync(0xffffffffu, lim < L::kBN)) {
          tmem_ld_32x32b_x32(s_addr, *reinterpret_cast<uint32_t(*)[32]>(&u[0]));
          tmem_ld_32x32b_x32(s_addr + 32, *reinterpret_cast<uint32_t(*)[32]>(&u[32]));
          tmem_wait_ld();
          regs_ready(*reinterpret_cast<uint32_t(*)[32]>(&u[0]));
          regs_ready(*reinterpret_cast<uint32_t(*)[32]>(&u[32]));
          tmem_ld_32x32b_x32(s_addr + 64, *reinterpret_cast<uint32_t(*)[32]>(&u[64]));
          tmem_ld_32x32b_x32(s_addr + 96, *reinterpret_cast<uint32_t(*)[32]>(&u[96]));
          const float neg_m0 = -m_run;
          float mxa = -INFINITY, mxb = -INFINITY;
          float sum0 = 0.f, sum1 = 0.f;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            if (q == 2) {
              tmem_wait_ld();
              regs_ready(*reinterpret_cast<uint32_t(*)[32]>(&u[64]));
              regs_ready(*reinterpret_cast<uint32_t(*)[32]>(&u[96]));
            }
            uint32_t pk[16];
#pragma unroll
            for (int e = 0; e < 32; e += 2) {
              const float s0 = __uint_as_float(u[q * 32 + e]), s1 = __uint_as_float(u[q * 32 + e + 1]);
              if (e & 2) mxb = fmax3(mxb, s0, s1); else mxa = fmax3(mxa, s0, s1);
              const float p0 = ex2_approx(fmaf(s0, scale_log2, neg_m0));
              const float p1 = ex2_approx(fmaf(s1, scale_log2, neg_m0));
              sum0 += p0;
              sum1 += p1;
              pk[e >> 1] = pack_bf16x2(p0, p1);
            }
            tmem_st_32x32b_x16(s_addr + q * 16, pk);
          }
          const float m_tile = fmaxf(mxa, mxb) * scale_log2;
          const bool move = m_tile > m_run + L::kSpecRedoThreshold;
          float alpha = 1.0f;
          if (__any_sync(0xffffffffu, move)) {  // redo the tile against the new max
            alpha = move ? ex2_approx(m_run - m_tile) : 1.0f;
            if (move) m_run = m_tile;
            const float neg_m = -m_run;
            sum0 = 0.f;
            sum1 = 0.f;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              uint32_t pk[16];
#pragma unroll
              for (int e = 0; e < 32; e += 2) {
                const float p0 = ex2_approx(fmaf(__uint_as_float(u[q * 32 + e]), scale_log2, neg_m));
                const float p1 = ex2_approx(fmaf(__uint_as_float(u[q * 32 + e + 1]), scale_log2, neg_m));
                sum0 += p0;
                sum1 += p1;
                pk[e >> 1] = pack_bf16x2(p0, p1);
              }
              tmem_st_32x32b_x16(s_addr + q * 16, pk);
            }
            if (!o_current()) {
              ok = false;
              break;
            }
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
              uint32_t v[32];
              tmem_ld_32x32b_x32(o_addr + c * 32, v);
              tmem_wait_ld_regs(v);
#pragma unroll
              for (int i2 = 0; i2 < 32; ++i2) v[i2] = __float_as_uint(__uint_as_float(v[i2]) * alpha);
              tmem_st_32x32b_x32(o_addr + c * 32, v);
            }
          }
          l_run = l_run * alpha + (sum0 + sum1);
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(bar(L::kPFull + sr.buf));
          continue;
        }
        // The same for a masked tile (the causal diagonal, keys past N): a
        // masked key's score becomes -inf, so its probability is exactly 0
        // and it never sets the max (the scale is positive here: a zero or
        // subnormal scale arrives as 1e-30).
        if (jj > 0 && !neg_scale && __any_sync(0xffffffffu, lim < L::kBN)) {
          tmem_ld_32x32b_x32(s_addr, *reinterpret_cast<uint32_t(*)[32]>(&u[0]));
          tmem_ld_32x32b_x32(s_addr + 32, *reinterpret_cast<uint32_t(*)[32]>(&u[32]));
          tmem_wait_ld();
          regs_ready(*reinterpret_cast<uint32_t(*)[32]>(&u[0]));
          regs_ready(*reinterpret_cast<uint32_t(*)[32]>(&u[32]));
          tmem_ld_32x32b_x32(s_addr + 64, *reinterpret_cast<uint32_t(*)[32]>(&u[64]));
          tmem_ld_32x32b_x32(s_addr + 96, *reinterpret_cast<uint32_t(*)[32]>(&u[96]));
#pragma unroll
          for (int c = 0; c < 64; ++c) u[c] = (c < lim) ? u[c] : masked_bits;
          const float neg_m0 = -m_run;
          float mxa = -INFINITY, mxb = -INFINITY;
          float sum0 = 0.f, sum1 = 0.f;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            if (q == 2) {
              tmem_wait_ld();
              regs_ready(*reinterpret_cast<uint32_t(*)[32]>(&u[64]));
              regs_ready(*reinterpret_cast<uint32_t(*)[32]>(&u[96]));
#pragma unroll
              for (int c = 64; c < 128; ++c) u[c] = (c < lim) ? u[c] : masked_bits;
            }
            uint32_t pk[16];
#pragma unroll
            for (int e = 0; e < 32; e += 2) {
              const float s0 = __uint_as_float(u[q * 32 + e]), s1 = __uint_as_float(u[q * 32 + e + 1]);
              if (e & 2) mxb = fmax3(mxb, s0, s1); else mxa = fmax3(mxa, s0, s1);
              const float p0 = ex2_approx(fmaf(s0, scale_log2, neg_m0));
              const float p1 = ex2_approx(fmaf(s1, scale_log2, neg_m0));
              sum0 += p0;
              sum1 += p1;
              pk[e >> 1] = pack_bf16x2(p0, p1);
            }
            tmem_st_32x32b_x16(s_addr + q * 16, pk);
          }
          const float m_tile = fmaxf(mxa, mxb) * scale_log2;
          const bool move = m_tile > m_run + L::kSpecRedoThreshold;
          float alpha = 1.0f;
          if (__any_sync(0xffffffffu, move)) {  // redo the tile against the new max
            alpha = move ? ex2_approx(m_run - m_tile) : 1.0f;
            if (move) m_run = m_tile;
            const float neg_m = -m_run;
            sum0 = 0.f;
            sum1 = 0.f;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              uint32_t pk[16];
#pragma unroll
              for (int e = 0; e < 32; e += 2) {
                const float p0 = ex2_approx(fmaf(__uint_as_float(u[q * 32 + e]), scale_log2, neg_m));
                const float p1 = ex2_approx(fmaf(__uint_as_float(u[q * 32 + e + 1]), scale_log2, neg_m));
                sum0 += p0;
                sum1 += p1;
                pk[e >> 1] = pack_bf16x2(p0, p1);
              }
              tmem_st_32x32b_x16(s_addr + q * 16, pk);
            }
            if (!o_current()) {
              ok = false;
              break;
            }
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
              uint32_t v[32];
              tmem_ld_32x32b_x32(o_addr + c * 32, v);
              tmem_wait_ld_regs(v);
#pragma unroll
              for (int i2 = 0; i2 < 32; ++i2) v[i2] = __float_as_uint(__uint_as_float(v[i2]) * alpha);
              tmem_st_32x32b_x32(o_addr + c * 32, v);
            }
          }
          l_run = l_run * alpha + (sum0 + sum1);
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(bar(L::kPFull + sr.buf));
          continue;
        }
#pragma unroll
        for (int c = 0; c < 4; ++c)
          tmem_ld_32x32b_x32(s_addr + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&u[c * 32]));
        tmem_wait_ld_regs(u);
        // mask: causal diagonal tile (key > query) and keys past the end.  A
        // masked score becomes the value that scales to -inf.
        if (lim < L::kBN) {
#pragma unroll
          for (int c = 0; c < 128; ++c) u[c] = (c < lim) ? u[c] : masked_bits;
        }
        // row max of scale*log2(e)*s: the max of s, or its min for a negative scale
        float mx0 = __uint_as_float(u[0]), mx1 = __uint_as_float(u[1]);
        float mx2 = __uint_as_float(u[2]), mx3 = __uint_as_float(u[3]);
        if (neg_scale) {
#pragma unroll
          for (int c = 4; c < 128; c += 8) {
            mx0 = fmin3(mx0, __uint_as_float(u[c]), __uint_as_float(u[c + 1]));
            mx1 = fmin3(mx1, __uint_as_float(u[c + 2]), __uint_as_float(u[c + 3]));
            mx2 = fmin3(mx2, __uint_as_float(u[c + 4]), __uint_as_float(u[c + 5]));
            mx3 = fmin3(mx3, __uint_as_float(u[c + 6]), __uint_as_float(u[c + 7]));
          }
          mx0 = fminf(fmin3(mx0, mx1, mx2), mx3);
        } else {
#pragma unroll
          for (int c = 4; c < 128; c += 8) {
            mx0 = fmax3(mx0, __uint_as_float(u[c]), __uint_as_float(u[c + 1]));
            mx1 = fmax3(mx1, __uint_as_float(u[c + 2]), __uint_as_float(u[c + 3]));
            mx2 = fmax3(mx2, __uint_as_float(u[c + 4]), __uint_as_float(u[c + 5]));
            mx3 = fmax3(mx3, __uint_as_float(u[c + 6]), __uint_as_float(u[c + 7]));
          }
          mx0 = fmaxf(fmax3(mx0, mx1, mx2), mx3);
        }
        const float m_tile = mx0 * scale_log2;
        const bool move = m_tile > m_run + L::kRescaleThreshold;
        const float alpha = move ? ex2_approx(m_run - m_tile) : 1.0f;
        if (move) m_run = m_tile;
        const float neg_m = -m_run;
        float sum0 = 0.f, sum1 = 0.f;
        // warp-uniform branch: both paths end in tcgen05.st, which every lane of
        // the warp must execute together (a lane with lim == 128 masks nothing)
        if (__any_sync(0xffffffffu, lim < L::kBN)) {
          // masked tile: a masked key's probability is exactly 0 (also for a
          // zero scale, where the -inf * 0 product would not be -inf)
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint32_t pk[16];
#pragma unroll
            for (int e = 0; e < 32; e += 2) {
              const int c = q * 32 + e;
              float p0 = ex2_approx(fmaf(__uint_as_float(u[c]), scale_log2, neg_m));
              float p1 = ex2_approx(fmaf(__uint_as_float(u[c + 1]), scale_log2, neg_m));
              p0 = (c < lim) ? p0 : 0.f;
              p1 = (c + 1 < lim) ? p1 : 0.f;
              sum0 += p0;
              sum1 += p1;
              pk[e >> 1] = pack_bf16x2(p0, p1);
            }
            tmem_st_32x32b_x16(s_addr + q * 16, pk);
          }
        } else {
#pragma unroll
          for (int q = 0; q < 4; ++q) {  // 32 keys -> 16 packed bf16 pairs -> TMEM
            uint32_t pk[16];
#pragma unroll
            for (int e = 0; e < 32; e += 2) {
              const float a0 = fmaf(__uint_as_float(u[q * 32 + e]), scale_log2, neg_m);
              const float a1 = fmaf(__uint_as_float(u[q * 32 + e + 1]), scale_log2, neg_m);
              const float p0 = ex2_approx(a0);
              const float p1 = ex2_approx(a1);
              sum0 += p0;
              sum1 += p1;
              pk[e >> 1] = pack_bf16x2(p0, p1);
            }
            tmem_st_32x32b_x16(s_addr + q * 16, pk);
          }
        }
        l_run = l_run * alpha + (sum0 + sum1);
        if (jj > 0 && __any_sync(0xffffffffu, move)) {
          if (!o_current()) {
            ok = false;
            break;
          }
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t u[32];
            tmem_ld_32x32b_x32(o_addr + c * 32, u);
            tmem_wait_ld_regs(u);
#pragma unroll
            for (int i = 0; i < 32; ++i) u[i] = __float_as_uint(__uint_as_float(u[i]) * alpha);
            tmem_st_32x32b_x32(o_addr + c * 32, u);
          }
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(L::kPFull + sr.buf));
      }
      if (!ok) break;
      s_base += w.n0 + w.n1;

      // ---------------------------------------------------------- epilogue
      // the final O_t is complete once the tile's last P V is; it is read out
      // of TMEM before this warp group arrives on the next item's P, which is
      // what the next item's first P V (overwriting O_t) waits for
      if (n_t > 0) {
        if (!wait_bounded_warp(bar(L::kOFinal + t), of_cnt & 1, limit_ns, abort_flag,
                               err_fwd | kErrRoleEpilogue)) {
          ok = false;
          break;
        }
        ++of_cnt;
        tc_fence_after();
      }
      if (kSplit) {
        // partial result of this split for a real Q tile
        if (active) {
          const size_t tile_idx =
              (static_cast<size_t>(w.split) * bh_count + w.bh) * n_kv_all + qt;
          if (!dbg_check(tile_idx < static_cast<size_t>(num_splits) * bh_count * n_kv_all, err,
                         abort_flag))
            break;
          float* po = part_o + tile_idx * 128 * D + r * 4;
          if (n_t > 0) {
            const float inv_l = 1.0f / l_run;
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
              uint32_t u[32];
              tmem_ld_32x32b_x32(o_addr + c * 32, u);
              tmem_wait_ld_regs(u);
#pragma unroll
              for (int g = 0; g < 8; ++g)
                *reinterpret_cast<float4*>(po + (c * 8 + g) * 512) = make_float4(
                    __uint_as_float(u[4 * g]) * inv_l, __uint_as_float(u[4 * g + 1]) * inv_l,
                    __uint_as_float(u[4 * g + 2]) * inv_l, __uint_as_float(u[4 * g + 3]) * inv_l);
            }
          } else {
#pragma unroll
            for (int g = 0; g < D / 4; ++g)
              *reinterpret_cast<float4*>(po + g * 512) = make_float4(0.f, 0.f, 0.f, 0.f);
          }
          part_lse[tile_idx * 128 + r] = (n_t > 0) ? m_run + __log2f(l_run) : -INFINITY;
        }
      } else if (active) {
        // O_t / l as bf16: per 32 columns each thread writes its row's 64 bytes
        // into the warp's staging box (64-byte swizzle: 16-byte chunk q of row
        // r at chunk q ^ ((r >> 1) & 3), so the 8 rows of a shared-memory
        // wavefront hit distinct banks) and one lane stores the 32 x 32 box
        // with TMA (rows >= N clipped).  The box's earlier store, two boxes
        // back, must have finished reading it first.
        const float inv_l = 1.0f / l_run;
        const int row0 = qt * L::kBM + (warp & 3) * 32;  // first row of this warp's box
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t u[32];
          tmem_ld_32x32b_x32(o_addr + c * 32, u);
          tmem_wait_ld_regs(u);
          const uint32_t buf =
              sb + L::kOffStage + static_cast<uint32_t>((sw * 2 + (st_cnt & 1)) * L::kStageBytes);
          if (lane == 0) bulk_wait_group_read_1();
          __syncwarp();
#pragma unroll
          for (int q = 0; q < 4; ++q)
            st_shared_v4(buf + lane * 64 + ((q ^ ((lane >> 1) & 3)) << 4),
                         pack_bf16x2(__uint_as_float(u[8 * q + 0]) * inv_l,
                                     __uint_as_float(u[8 * q + 1]) * inv_l),
                         pack_bf16x2(__uint_as_float(u[8 * q + 2]) * inv_l,
                                     __uint_as_float(u[8 * q + 3]) * inv_l),
                         pack_bf16x2(__uint_as_float(u[8 * q + 4]) * inv_l,
                                     __uint_as_float(u[8 * q + 5]) * inv_l),
                         pack_bf16x2(__uint_as_float(u[8 * q + 6]) * inv_l,
                                     __uint_as_float(u[8 * q + 7]) * inv_l));
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            if (row0 < n) tma_store_3d(&tm_o, buf, c * 32, row0, w.bh);
            bulk_commit_group();
          }
          ++st_cnt;
        }
        const int row = qt * L::kBM + r;
        if (row < n)
          lse_out[static_cast<size_t>(w.bh) * n + row] =
              (m_run + __log2f(l_run)) * 0.69314718055994530942f;
      }
    }
    // the staging boxes must be read out before the CTA's shared memory goes
    if (lane == 0) bulk_wait_group_read_0();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, L::kTmemCols);
  }
  if (threadIdx.x == 0) sched_finish(sched_slot);
}

// Merge of the split partial results, page "FlashAttention 为什么能节省显存并提速,
// 是否改变注意力结果?", section 难点在于分块后softmax如何归一: blocks are brought to a
// common max before they are added.  With LSE_s = m_s + log2 l_s and
// O_s = u_s / l_s (base 2):  M = max_s LSE_s,  w_s = 2^(LSE_s - M)
// (= 2^(m_s - M) l_s),  l = sum_s w_s,  O = sum_s w_s O_s / l
// (= sum_s 2^(m_s - M) u_s / l),  LSE = M + log2 l, stored as natural log.
// Thread (p, row) owns 8 columns of one row; consecutive threads take
// consecutive rows so the partial reads are coalesced.
template <int D>
__global__ void __launch_bounds__(256)
    splitkv_combine_kernel(const float* __restrict__ part_o, const float* __restrict__ part_lse,
                           __nv_bfloat16* __restrict__ o, float* __restrict__ lse, int bh_count,
                           int n, int num_splits) {
  const long long idx = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const long long rows = static_cast<long long>(bh_count) * n;
  if (idx >= rows * (D / 8)) return;
  const int p = static_cast<int>(idx / rows);
  const long long row = idx % rows;
  const long long bh = row / n;
  const int r = static_cast<int>(row % n);
  const int n_tiles = (n + 127) / 128;
  const size_t tiles_per_split = static_cast<size_t>(bh_count) * n_tiles;
  const size_t tile = static_cast<size_t>(bh) * n_tiles + r / 128;
  float m = -INFINITY;
  for (int s = 0; s < num_splits; ++s)
    m = fmaxf(m, part_lse[(s * tiles_per_split + tile) * 128 + r % 128]);
  float l = 0.f;
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  for (int s = 0; s < num_splits; ++s) {
    const size_t t = s * tiles_per_split + tile;
    const float ls = part_lse[t * 128 + r % 128];
    if (ls == -INFINITY) continue;  // this split saw no key of the row
    const float w = ex2_approx(ls - m);
    l += w;
    const float* po = part_o + t * 128 * D + (r % 128) * 4;
    const float4 a = *reinterpret_cast<const float4*>(po + (2 * p) * 512);
    const float4 b = *reinterpret_cast<const float4*>(po + (2 * p + 1) * 512);
    acc[0] = fmaf(w, a.x, acc[0]);
    acc[1] = fmaf(w, a.y, acc[1]);
    acc[2] = fmaf(w, a.z, acc[2]);
    acc[3] = fmaf(w, a.w, acc[3]);
    acc[4] = fmaf(w, b.x, acc[4]);
    acc[5] = fmaf(w, b.y, acc[5]);
    acc[6] = fmaf(w, b.z, acc[6]);
    acc[7] = fmaf(w, b.w, acc[7]);
  }
  const float inv = 1.0f / l;
  uint4 out;
  out.x = pack_bf16x2(acc[0] * inv, acc[1] * inv);
  out.y = pack_bf16x2(acc[2] * inv, acc[3] * inv);
  out.z = pack_bf16x2(acc[4] * inv, acc[5] * inv);
  out.w = pack_bf16x2(acc[6] * inv, acc[7] * inv);
  *reinterpret_cast<uint4*>(o + row * D + 8 * p) = out;
  if (p == 0) lse[row] = (m + __log2f(l)) * 0.69314718055994530942f;
}

}  // namespace fa
