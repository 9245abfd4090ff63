// bwd_main.cuh -- main backward kernel: work item = (batch*head, 128-key tile).
//
// K_j and V_j stay in shared memory for the whole item; the Q tiles i that
// see key tile j (all of them, or i >= j under the causal mask, since Br = Bc)
// stream through a two-stage ring, dO_i through its own ring.  Per Q tile,
// with keys on the TMEM lanes (M = 128 keys):
//
//   S'^T  = K_j Q_i^T  - 1 (LSE2_i / c)^T     tcgen05 (c = scale * log2 e)
//   dP'^T = V_j dO_i^T - 1 D_i^T              tcgen05
//   P^T   = 2^(c S'^T)      one thread per key row, masked, written back over
//                           S'^T in TMEM as bf16
//   dV_j += P^T dO_i        tcgen05, A = P^T (TMEM), B = dO_i (MN-major)
//   dS^T  = P^T o dP'^T     written to shared memory as bf16
//   dK_j += dS^T Q_i        tcgen05, A = dS^T (K-major), B = Q_i (MN-major)
//   dQ_i  = dS K_j          tcgen05, A = dS^T read MN-major, B = K_j (MN-major)
//
// The per-query terms -LSE2_i / c and -D_i enter the two recompute GEMMs as
// one extra K = 16 step: A is a constant slab whose first three columns are
// 1, B a per-Q-tile slab holding the value split into three bf16 parts
// (hi + mid + lo carries it to about fp32 accuracy).  The tensor core thus
// does the per-column subtraction and the softmax threads load no per-column
// values.  Warp 2 builds those slabs from LSE2 and D in global memory.
//
// Issue order of the tensor-core work: ... dV_i, S_{i+1}, dQ_i, dK_i, dP_{i+1},
// dV_{i+1} ...  S_{i+1} goes right after dV_i (tcgen05.mma ops of one thread
// run in order, so it cannot overwrite P_i before dV_i has read it), which lets
// the exponentials of tile i+1 overlap dQ_i and dK_i on the tensor core; dQ_i
// goes before dK_i so that its read-out overlaps dK_i and dP_{i+1}, which
// reuses its TMEM columns, is not held up.
//
// The kernel is persistent: about one CTA per SM, each taking items until
// none are left (the first from blockIdx.x, the rest from a per-launch work
// counter).  The Q / dO rings and every barrier phase run on across items, so
// the next item's first Q and dO tiles load while the current item's last
// tiles are computed, its K_j / V_j load as soon as the last MMAs that read
// the current ones are done (prefetched into L2 when the item is claimed),
// and the compute warps store the current item's dK_j, dV_j while the next
// item's first scores are computed.  With one CTA per item, a CTA's fixed
// costs (set-up, first loads, pipeline fill and drain, epilogue) were paid
// once per key tile, which dominated short sequences (B=128 H=16 N=512 causal:
// about 17k cycles per CTA against 5.6k per Q tile).
//
// dK_j and dV_j accumulate in TMEM and are written once per item (no
// atomics): each compute warp converts its 32 key rows to bf16 through
// 32 x 32 staging boxes (64-byte swizzle; two per warp with four compute
// warps, one with eight) that one lane stores with TMA.  dQ_i partial
// products are read out of TMEM (by a separate warp group at d = 128) and
// added into the fp32 accumulator with vector atomic adds.  The accumulator
// keeps each 128-row tile as [D/4 column groups][128 rows][4 floats] so that
// those adds are coalesced.  For d = 128 the 64 KB of adds of one Q tile are paced,
// an 80 ns sleep after each pair of vector adds (about 1.3 us in all, under
// half of a Q-loop iteration): issued as one burst they queue ahead of the
// next tile loads and stretch every iteration (B200: 857 -> 940 TFLOP/s for
// this kernel at B=2 H=16 N=4096, 880-930 -> 988 at B=1 H=32 N=16384).
// Sleeping for most of the iteration instead (2.4 us) makes the read-out fall
// behind, and dP of the tile after next waits for it: 650 TFLOP/s.  For
// d = 64 pacing measured slightly slower.
//
// Warp roles (384 threads): warp 0 TMA producer and scheduler; warp 1 TMEM
// allocator and MMA issuer; warp 2 builds the LSE / D slabs; warps 4-7
// compute P^T / dS^T (thread = key row) and write dK, dV; at d = 128 warps
// 8-11 read dQ out of TMEM (thread = query row) and add it to global.
// Without dQ (the deterministic backward), and with dQ at d = 64, warps 8-11
// instead share the P^T / dS^T work: each warp group takes 64 of the 128
// query columns (and the same half of the columns of dK, dV and dQ, whose
// read-out the two groups then do between a tile's P^T and its dS^T).  At
// d = 128 dQ reuses dP'^T's TMEM columns, so the next dP waits for its
// read-out, which only a warp group of its own does at once (the compute
// warps doing it: B=2 H=16 N=4096 -8 %); at d = 64 dQ has columns of its own
// and the shared work pays (B=16 H=16 N=4096 +11 %, B=64 H=16 N=1024 +16 %).
// P^T of query half h sits in the first 32 of the 64 TMEM columns S'^T had
// for those queries.
//
// TMEM columns:  dK [0,D), dV [D,2D), S'^T/P^T [2D,2D+128), dP'^T [2D+128,2D+256);
// at d = 128 dQ reuses the dP'^T columns once dS^T has been formed (all 512
// are taken), at d = 64 it has [384, 448).
#pragma once

namespace fa {

template <int D>
struct BwdLayout {
  static constexpr int kThreads = 384;
  static constexpr int kTile = 128 * D * 2;   // bytes of a K, V, Q or dO tile
  static constexpr int kSq = 128 * 128 * 2;   // bytes of the bf16 dS^T tile
  static constexpr int kSlab = 128 * 16 * 2;  // bytes of a 128 x 16 bf16 slab
  static constexpr int kDoStages = (D == 64) ? 2 : 1;
  static constexpr int kBox = 32 * 32 * 2;    // one 32 x 32 bf16 dK / dV staging box
  static constexpr int kOffK = 0;
  static constexpr int kOffV = kOffK + kTile;
  static constexpr int kOffQ = kOffV + kTile;                // [2]
  static constexpr int kOffDO = kOffQ + 2 * kTile;           // [kDoStages]
  static constexpr int kOffDS = kOffDO + kDoStages * kTile;
  static constexpr int kOffOnes = kOffDS + kSq;              // constant A slab
  static constexpr int kOffQSlab = kOffOnes + kSlab;         // [2] -LSE2/c parts
  static constexpr int kOffDoSlab = kOffQSlab + 2 * kSlab;   // [kDoStages] -D parts
  // 8 boxes: two per compute warp with dQ (4 warps), one without (8 warps)
  static constexpr int kOffStage = kOffDoSlab + kDoStages * kSlab;
  static constexpr int kOffBar = kOffStage + 8 * kBox;
  static constexpr int kBarArea = 256;
  static constexpr int kBytes = kOffBar + kBarArea;
  static constexpr int kSmemAlloc = kBytes + 1024;  // slack to align the base to 1 KiB
  static_assert(kSmemAlloc <= 232448, "shared memory budget");
  static_assert(kOffStage % 512 == 0, "64-byte swizzle atoms of the staging boxes");
  // barriers
  static constexpr int kKvFull = 0, kQFull = 1 /*[2]*/, kQEmpty = 3 /*[2]*/, kDoFull = 5 /*[2]*/,
                       kDoEmpty = 7 /*[2]*/, kSFull = 9, kPReady = 10, kDpFull = 11,
                       kDsReady = 12, kDsFree = 13, kDqFull = 14, kDqFree = 15, kDkdvDone = 16,
                       kDrain = 17, kKvEmpty = 18, kDkdvFree = 19, kItemFull = 20 /*[2]*/,
                       kItemEmpty = 22 /*[2]*/, kNumBars = 24;
  // readers of the item ring: warps 1, 2 and 4-11
  static constexpr int kItemReaders = 10;
  static constexpr int kOffSlot = kOffBar + 8 * kNumBars;
  static constexpr int kOffAbort = kOffSlot + 4;
  static constexpr int kOffItems = kOffAbort + 4;  // int[2]
  static_assert(kOffItems + 8 <= kOffBar + kBarArea, "barrier area too small");
  // TMEM columns
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kColDK = 0;
  static constexpr uint32_t kColDV = D;
  static constexpr uint32_t kColS = 2 * D;
  static constexpr uint32_t kColDP = 2 * D + 128;
  // d = 128 fills all 512 columns, so dQ reuses dP'^T's once dS^T is formed;
  // at d = 64 it has columns of its own
  static constexpr bool kDqOwnCols = (D == 64);
  static constexpr uint32_t kColDQ = kDqOwnCols ? kColDP + 128 : kColDP;
  static_assert(kColDP + 128 <= kTmemCols && kColDQ + D <= kTmemCols, "TMEM budget");
};

// Shared-memory descriptor of a 128 x 16 bf16 K-major slab with 32-byte
// swizzle: row r at 32 r bytes, its two 16-byte halves swapped when bit 2 of r
// is set; SBO = 256 bytes between 8-row groups; layout type 6.
__device__ __forceinline__ uint64_t sw32_slab_desc(uint32_t saddr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>(1) << 16;         // LBO (unused): 16 bytes
  d |= static_cast<uint64_t>(256 >> 4) << 32;  // SBO
  d |= static_cast<uint64_t>(1) << 46;
  d |= static_cast<uint64_t>(6) << 61;
  return d;
}

// Writes row r of a slab: columns 0..2 hold v0, v1, v2 (bf16), the rest 0.
__device__ __forceinline__ void slab_row(uint32_t slab, int r, float v0, float v1, float v2) {
  const uint32_t lo = pack_bf16x2(v0, v1), hi = pack_bf16x2(v2, 0.f);
  const uint32_t swz = static_cast<uint32_t>((r >> 2) & 1);
  st_shared_v4(slab + r * 32 + (swz << 4), lo, hi, 0u, 0u);          // columns 0..7
  st_shared_v4(slab + r * 32 + ((swz ^ 1u) << 4), 0u, 0u, 0u, 0u);  // columns 8..15
}

// x as three bf16-exact parts a + b + c (each part the bf16 rounding of the
// remainder, so the sum matches x to about 2^-24 relative).
__device__ __forceinline__ void split3(float x, float& a, float& b, float& c) {
  a = __bfloat162float(__float2bfloat16_rn(x));
  const float r1 = x - a;
  b = __bfloat162float(__float2bfloat16_rn(r1));
  c = __bfloat162float(__float2bfloat16_rn(r1 - b));
}

// kDq = false (deterministic backward): no dQ MMA and no atomics here; dQ
// comes from dq_pass_kernel.  dP_{i+1} then only waits for dS_i to be formed.
// pause after each pair of dQ vector adds (d = 128)
constexpr uint32_t kAddGapNs = 80;

// Work item `lin` -> (head, key tile).  Items run in groups of `hg` heads
// (chosen by the host from the heads' L2 footprint), and within a group key
// tile 0 of every head first, then key tile 1, ... (small j = the longest
// loop under the causal mask).  The CTAs busy at any time then share the Q,
// dO and dQ accumulator tiles of a few heads, which stay in L2, and the last
// items of a launch are short ones.
struct BwdItem {
  int bh, j, i0, n_it;
};
template <bool kCausal>
__device__ __forceinline__ BwdItem bwd_item(int lin, int n_kt, int bh_count, int hg) {
  const int grp = lin / (hg * n_kt);
  const int g_base = grp * hg;
  const int g_size = min(hg, bh_count - g_base);
  const int g_off = lin - grp * hg * n_kt;
  BwdItem w;
  w.bh = g_base + g_off % g_size;
  w.j = g_off / g_size;
  w.i0 = kCausal ? w.j : 0;
  w.n_it = n_kt - w.i0;
  return w;
}

template <int D, bool kCausal, bool kDq>
__global__ void __launch_bounds__(384, 1)
    bwd_main_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                    const __grid_constant__ CUtensorMap tm_dk, const __grid_constant__ CUtensorMap tm_dv,
                    const float* __restrict__ dvec, const float* __restrict__ lse2,
                    float* __restrict__ dq_acc, int n, int np, float scale, float c_exp,
                    uint64_t limit_ns, int bh_count, int n_items, uint32_t sched_slot,
                    int head_group) {
  using L = BwdLayout<D>;
  constexpr int kDBlk = D / 64;
  constexpr int DS = L::kDoStages;
  // With dQ at d = 64 (own TMEM columns) all eight compute warps share the
  // P^T / dS^T work by query halves and read dQ out themselves; at d = 128
  // warps 4-7 compute and warps 8-11 read dQ out (its columns are dP'^T's,
  // so the next dP waits for the read-out, which a separate warp group does
  // at once).
  constexpr bool kSplitDq = kDq && L::kDqOwnCols;
  constexpr bool kEight = !kDq || kSplitDq;  // eight compute warps

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
  const int n_kt = np / 128;  // key tiles = query tiles
  const unsigned int err_k = kErrBwdMain;

  if (threadIdx.x == 0) {
    for (int b = 0; b < L::kNumBars; ++b) {
      uint32_t cnt = 1;
      if (b == L::kDqFree) cnt = 4;  // the dQ read-out warps
      if (b == L::kPReady || b == L::kDsReady || b == L::kDkdvFree)
        cnt = kEight ? 8 : 4;  // the compute warps
      if ((b >= L::kQFull && b < L::kQFull + 2) || (b >= L::kDoFull && b < L::kDoFull + 2))
        cnt = 2;  // the TMA producer and the slab builder
      if (b == L::kItemEmpty || b == L::kItemEmpty + 1) cnt = L::kItemReaders;
      mbar_init(bar(b), cnt);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (threadIdx.x < 128) {  // constant A slab: 1 in the first three columns
    slab_row(sb + L::kOffOnes, threadIdx.x, 1.f, 1.f, 1.f);
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

  // Ring positions: an item's Q tiles are numbered on from the tiles of the
  // CTA's earlier items (t = tiles before + it); Q_t sits in stage t & 1,
  // dO_t in stage t % DS, and every per-tile barrier completes once per t.
  if (warp == 0) {
    // --------------------------------------------------- producer, scheduler
    const uint32_t err = err_k | kErrRoleLoad;
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      tma_prefetch_desc(&tm_do);
    }
    int gq = 0;                // Q tiles of the earlier items
    int nq = 0, ndo = 0, nkv = 0;  // loads issued (for the drain)
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
      const BwdItem w = bwd_item<kCausal>(item, n_kt, bh_count, head_group);
      bool ok = true;
      if (lane == 0) {
        // a failed check raises the abort flag; the other roles then give up
        ok = dbg_check(w.j * 128 < n && w.bh >= 0 && w.bh < bh_count && w.i0 + w.n_it <= n_kt,
                       err, abort_flag);
        // order: Q_0, dO_0 (their stages free up first), K_j / V_j (once the
        // previous item's MMAs no longer read K and V), then the other tiles
        for (int it = 0; ok && it < w.n_it; ++it) {
          const int t = gq + it;
          const int i = w.i0 + it;
          const int st = t & 1;
          if (!dbg_check(i * 128 < n, err, abort_flag) ||
              !wait_bounded(bar(L::kQEmpty + st), ((t >> 1) & 1) ^ 1, limit_ns, abort_flag, err)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(bar(L::kQFull + st), L::kTile);
          for (int db = 0; db < kDBlk; ++db)
            tma_load_3d(sb + L::kOffQ + st * L::kTile + db * 16384, &tm_q, bar(L::kQFull + st),
                        db * 64, i * 128, w.bh);
          ++nq;
          const int ds = t % DS;
          if (!wait_bounded(bar(L::kDoEmpty + ds), ((t / DS) & 1) ^ 1, limit_ns, abort_flag, err)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(bar(L::kDoFull + ds), L::kTile);
          for (int db = 0; db < kDBlk; ++db)
            tma_load_3d(sb + L::kOffDO + ds * L::kTile + db * 16384, &tm_do, bar(L::kDoFull + ds),
                        db * 64, i * 128, w.bh);
          ++ndo;
          if (it == 0) {
            if (k > 0 && !wait_bounded(bar(L::kKvEmpty), (k - 1) & 1, limit_ns, abort_flag, err)) {
              ok = false;
              break;
            }
            mbar_arrive_expect_tx(bar(L::kKvFull), 2 * L::kTile);
            for (int db = 0; db < kDBlk; ++db) {
              tma_load_3d(sb + L::kOffK + db * 16384, &tm_k, bar(L::kKvFull), db * 64, w.j * 128,
                          w.bh);
              tma_load_3d(sb + L::kOffV + db * 16384, &tm_v, bar(L::kKvFull), db * 64, w.j * 128,
                          w.bh);
            }
            ++nkv;
          }
        }
      }
      if (__shfl_sync(0xffffffffu, ok ? 1 : 0, 0) == 0) break;
      gq += w.n_it;
      // claim the next item now that this one's loads are all issued, and
      // start its K_j / V_j on their way into L2
      unsigned int f = 0;
      if (lane == 0) f = atomicAdd(&g_sched_next[sched_slot], 1u);
      f = __shfl_sync(0xffffffffu, f, 0);
      item = f >= static_cast<unsigned int>(n_items) - gridDim.x ? -1
                                                                  : static_cast<int>(gridDim.x + f);
      if (lane == 0 && item >= 0) {
        const BwdItem nw = bwd_item<kCausal>(item, n_kt, bh_count, head_group);
        for (int db = 0; db < kDBlk; ++db) {
          tma_prefetch_l2_3d(&tm_k, db * 64, nw.j * 128, nw.bh);
          tma_prefetch_l2_3d(&tm_v, db * 64, nw.j * 128, nw.bh);
        }
      }
    }
    if (lane == 0 && *abort_flag) {
      // copies already issued must land before shared memory is released;
      // with the slab builder's arrival possibly missing, these waits may
      // run to their limit, which only delays the exit
      if (nkv > 0) drain_wait(bar(L::kKvFull), (nkv - 1) & 1, limit_ns);
      for (int t = (nq > 2 ? nq - 2 : 0); t < nq; ++t)
        drain_wait(bar(L::kQFull + (t & 1)), (t >> 1) & 1, limit_ns);
      for (int t = (ndo > DS ? ndo - DS : 0); t < ndo; ++t)
        drain_wait(bar(L::kDoFull + t % DS), (t / DS) & 1, limit_ns);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // the whole warp runs this loop; the MMA and commit wrappers elect one lane
    constexpr uint32_t id_kk = idesc_bf16_f32(128, 128, false, false);
    constexpr uint32_t id_kmn = idesc_bf16_f32(128, D, false, true);
    constexpr uint32_t id_mnmn = idesc_bf16_f32(128, D, true, true);
    // With dQ the MMA loops are unrolled only by 2, which keeps the hot code
    // of the MMA, compute and dQ warps that share a scheduler within its
    // instruction cache (B200, against full unrolling: no_instruction stalls
    // down, B=64 H=16 N=1024 causal +18 %, B=16 H=16 N=4096 d=64 +15 %;
    // against no unrolling: B=2 H=16 N=4096 +2 %).  Without dQ the tensor
    // pipe is the busier unit and full unrolling measured faster (B=2 H=16
    // N=4096: +8 %).
    constexpr int kMmaUnroll = (kDq && !kSplitDq) ? 2 : 8;
    const uint32_t err = err_k | kErrRoleMma;
    const uint32_t a_k = sb + L::kOffK, a_v = sb + L::kOffV, a_ds = sb + L::kOffDS;
    const uint64_t d_ones = sw32_slab_desc(sb + L::kOffOnes);
    auto issue_s = [&](int t) {  // S'^T = K_j Q_i^T - 1 (LSE2_i / c)^T
      const uint32_t a_q = sb + L::kOffQ + (t & 1) * L::kTile;
#pragma unroll kMmaUnroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
        mma_bf16_ss(tmem + L::kColS, sw128_desc(a_k + off, 16, 1024),
                    sw128_desc(a_q + off, 16, 1024), id_kk, kk > 0 ? 1u : 0u);
      }
      mma_bf16_ss(tmem + L::kColS, d_ones,
                  sw32_slab_desc(sb + L::kOffQSlab + (t & 1) * L::kSlab), id_kk, 1u);
      tc_commit(bar(L::kSFull));
    };
    auto issue_dp = [&](int t) {  // dP'^T = V_j dO_i^T - 1 D_i^T
      const int ds = t % DS;
      const uint32_t a_do = sb + L::kOffDO + ds * L::kTile;
#pragma unroll kMmaUnroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
        mma_bf16_ss(tmem + L::kColDP, sw128_desc(a_v + off, 16, 1024),
                    sw128_desc(a_do + off, 16, 1024), id_kk, kk > 0 ? 1u : 0u);
      }
      mma_bf16_ss(tmem + L::kColDP, d_ones,
                  sw32_slab_desc(sb + L::kOffDoSlab + ds * L::kSlab), id_kk, 1u);
      tc_commit(bar(L::kDpFull));
    };
    int gq = 0;
    for (int k = 0;; ++k) {
      int item = -1;
      if (!read_item(k, item, err) || item < 0) break;
      const BwdItem w = bwd_item<kCausal>(item, n_kt, bh_count, head_group);
      // the first dP overwrites the columns of the previous item's last dQ
      bool ok = wait_bounded_warp(bar(L::kKvFull), k & 1, limit_ns, abort_flag, err) &&
                wait_bounded_warp(bar(L::kQFull + (gq & 1)), (gq >> 1) & 1, limit_ns, abort_flag,
                                  err) &&
                wait_bounded_warp(bar(L::kDoFull + gq % DS), (gq / DS) & 1, limit_ns, abort_flag,
                                  err) &&
                (!kDq || kSplitDq || gq == 0 ||
                 wait_bounded_warp(bar(L::kDqFree), (gq - 1) & 1, limit_ns, abort_flag, err));
      if (!ok) break;
      tc_fence_after();
      issue_s(gq);
      issue_dp(gq);
      // the first dV and dK of an item overwrite the accumulators, which the
      // previous item's epilogue must have read (it has, long before P_0 of
      // this item is ready)
      if (k > 0 && !wait_bounded_warp(bar(L::kDkdvFree), (k - 1) & 1, limit_ns, abort_flag, err))
        break;
      for (int it = 0; ok && it < w.n_it; ++it) {
        const int t = gq + it;
        const uint32_t ph = t & 1;
        const int st = t & 1;
        const int ds = t % DS;
        const uint32_t a_q = sb + L::kOffQ + st * L::kTile;
        const uint32_t a_do = sb + L::kOffDO + ds * L::kTile;
        const bool next = it + 1 < w.n_it;
        if (!wait_bounded_warp(bar(L::kPReady), ph, limit_ns, abort_flag, err)) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll kMmaUnroll
        for (int kk = 0; kk < 8; ++kk)  // dV_j += P^T dO_i  (K = 128 queries, P^T in TMEM)
          mma_bf16_ts(tmem + L::kColDV, tmem + L::kColS + (kk >> 2) * 64 + (kk & 3) * 8,
                      sw128_desc(a_do + kk * 2048, 16384, 1024), id_kmn,
                      (it > 0 || kk > 0) ? 1u : 0u);
        tc_commit(bar(L::kDoEmpty + ds));  // dO_i and its slab are no longer read
        if (next) {  // S of the next Q tile, as soon as P_i has been consumed
          if (!wait_bounded_warp(bar(L::kQFull + ((t + 1) & 1)), ((t + 1) >> 1) & 1, limit_ns,
                                 abort_flag, err)) {
            ok = false;
            break;
          }
          tc_fence_after();
          issue_s(t + 1);
        }
        if (!wait_bounded_warp(bar(L::kDsReady), ph, limit_ns, abort_flag, err)) {
          ok = false;
          break;
        }
        tc_fence_after();
        // dQ_i first: its read-out (and the dP_{i+1} that reuses its columns)
        // then overlaps dK_i
        if (kDq) {
#pragma unroll kMmaUnroll
          for (int kk = 0; kk < 8; ++kk)  // dQ_i = dS K_j  (K = 128 keys)
            mma_bf16_ss(tmem + L::kColDQ, sw128_desc(a_ds + kk * 2048, 16384, 1024),
                        sw128_desc(a_k + kk * 2048, 16384, 1024), id_mnmn, kk > 0 ? 1u : 0u);
          tc_commit(bar(L::kDqFull));
        }
        // every MMA that reads K_j or V_j has been issued: the next item's
        // K and V may load once they are done
        if (!next) tc_commit(bar(L::kKvEmpty));
#pragma unroll kMmaUnroll
        for (int kk = 0; kk < 8; ++kk) {  // dK_j += dS^T Q_i
          const uint32_t acc = (it > 0 || kk > 0) ? 1u : 0u;
          if (kDq) {  // dS^T from shared memory (K-major)
            const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
            mma_bf16_ss(tmem + L::kColDK, sw128_desc(a_ds + off, 16, 1024),
                        sw128_desc(a_q + kk * 2048, 16384, 1024), id_kmn, acc);
          } else {  // dS^T from TMEM over dP'^T, laid out like P^T
            mma_bf16_ts(tmem + L::kColDK, tmem + L::kColDP + (kk >> 2) * 64 + (kk & 3) * 8,
                        sw128_desc(a_q + kk * 2048, 16384, 1024), id_kmn, acc);
          }
        }
        tc_commit(bar(L::kQEmpty + st));  // Q_i and its slab are no longer read
        tc_commit(bar(L::kDsFree));
        if (next) {  // dP of the next Q tile once dQ_i has left the shared columns
          if (kDq && !kSplitDq &&
              !wait_bounded_warp(bar(L::kDqFree), ph, limit_ns, abort_flag, err)) {
            ok = false;
            break;
          }
          if (!wait_bounded_warp(bar(L::kDoFull + (t + 1) % DS), ((t + 1) / DS) & 1, limit_ns,
                                 abort_flag, err)) {
            ok = false;
            break;
          }
          tc_fence_after();
          issue_dp(t + 1);
        }
      }
      if (!ok) break;
      tc_commit(bar(L::kDkdvDone));
      gq += w.n_it;
    }
    tc_commit(bar(L::kDrain));
    drain_wait(bar(L::kDrain), 0, limit_ns);
    __syncwarp();
  } else if (warp == 2) {
    // ------------------------------------------------------- slab builder
    // Q slab of tile i: row q holds -LSE2_q / c in three bf16 parts; dO slab:
    // -D_q in three parts.  Rows past the end of the sequence (LSE2 = +inf)
    // get a large finite value whose scaled exponential is 0.
    const uint32_t err = err_k | kErrRoleLoad;
    const float inv_c = 1.0f / c_exp;
    // c * pad = -200 (or beyond): its base-2 exponential is 0 in fp32
    const float pad = copysignf(fminf(200.0f / fabsf(c_exp), 3.0e38f), -c_exp);
    int gq = 0;
    bool ok = true;
    for (int k = 0; ok; ++k) {
      int item = -1;
      if (!read_item(k, item, err) || item < 0) break;
      const BwdItem w = bwd_item<kCausal>(item, n_kt, bh_count, head_group);
      for (int it = 0; it < w.n_it; ++it) {
        const int t = gq + it;
        const int i = w.i0 + it;
        const int st = t & 1;
        const size_t vrow = static_cast<size_t>(w.bh) * np + static_cast<size_t>(i) * 128 +
                            static_cast<size_t>(lane) * 4;
        if (!dbg_check(vrow + 4 <= static_cast<size_t>(bh_count) * np, err, abort_flag)) {
          ok = false;
          break;
        }
        const float4 l4 = *reinterpret_cast<const float4*>(lse2 + vrow);
        const float4 d4 = *reinterpret_cast<const float4*>(dvec + vrow);
        if (!wait_bounded_warp(bar(L::kQEmpty + st), ((t >> 1) & 1) ^ 1, limit_ns, abort_flag,
                               err)) {
          ok = false;
          break;
        }
        const float lv[4] = {l4.x, l4.y, l4.z, l4.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float x = (lv[e] == INFINITY) ? pad : -lv[e] * inv_c;
          float a, b, c;
          split3(x, a, b, c);
          slab_row(sb + L::kOffQSlab + st * L::kSlab, lane * 4 + e, a, b, c);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(L::kQFull + st));
        const int ds = t % DS;
        if (!wait_bounded_warp(bar(L::kDoEmpty + ds), ((t / DS) & 1) ^ 1, limit_ns, abort_flag,
                               err)) {
          ok = false;
          break;
        }
        const float dv[4] = {d4.x, d4.y, d4.z, d4.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          float a, b, c;
          split3(-dv[e], a, b, c);
          slab_row(sb + L::kOffDoSlab + ds * L::kSlab, lane * 4 + e, a, b, c);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(L::kDoFull + ds));
      }
      gq += w.n_it;
    }
  } else if (warp >= 4 && (warp < 8 || kEight)) {
    // ------------------------------------------------ P^T, dS^T, dK / dV out
    // four compute warps: warps 4-7 take all 128 query columns; eight: warps
    // 4-7 take queries 0-63 and warps 8-11 queries 64-127 (and the two halves
    // of the columns of dK, dV and, with dQ, dQ)
    constexpr int kHalves = kEight ? 1 : 2;
    constexpr int kBoxes = kEight ? 1 : 2;  // staging boxes of this warp
    const int h0 = kEight ? (warp >> 2) - 1 : 0;
    const int r = (warp & 3) * 32 + lane;  // key row in the tile == TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t err = err_k | kErrRoleSoftmax;
    const uint32_t dsrow = sb + L::kOffDS + r * 128;
    const uint32_t box0 = sb + L::kOffStage + static_cast<uint32_t>((warp - 4) * kBoxes * L::kBox);
    bool ok = dbg_check(tmem_range_ok(tmem + lane_off + L::kColDP, tmem, 128, L::kTmemCols) &&
                            tmem_range_ok(tmem + lane_off + L::kColDV, tmem, D, L::kTmemCols) &&
                            tmem_range_ok(tmem + lane_off + L::kColS, tmem, 128, L::kTmemCols),
                        err, abort_flag);
    // (eight compute warps with dQ) dQ of Q tile i, tile t of this CTA's
    // sequence: once its MMA is done this warp group reads its half of the
    // columns for the 128 query rows (thread = query row = TMEM lane) and adds
    // them into the fp32 accumulator, laid out as for the read-out warps below
    auto dq_out = [&](int t, int i, int bh) -> bool {
      if (!wait_bounded_warp(bar(L::kDqFull), t & 1, limit_ns, abort_flag, err_k | kErrRoleDq))
        return false;
      tc_fence_after();
      uint32_t u[D / 2];
#pragma unroll
      for (int cc = 0; cc < D / 64; ++cc)
        tmem_ld_32x32b_x32(tmem + lane_off + L::kColDQ + h0 * (D / 2) + cc * 32,
                           *reinterpret_cast<uint32_t(*)[32]>(&u[cc * 32]));
      tmem_wait_ld_regs(u);
      if (!dbg_check(static_cast<size_t>(bh) * n_kt + i < static_cast<size_t>(bh_count) * n_kt,
                     err_k | kErrRoleDq, abort_flag))
        return false;
      float* dst = dq_acc + (static_cast<size_t>(bh) * n_kt + static_cast<size_t>(i)) * 128 * D +
                   static_cast<size_t>(h0) * (D / 8) * 512 + static_cast<size_t>(r) * 4;
#pragma unroll
      for (int q = 0; q < D / 8; ++q)
        red_add_v4(dst + q * 512, __uint_as_float(u[4 * q]), __uint_as_float(u[4 * q + 1]),
                   __uint_as_float(u[4 * q + 2]), __uint_as_float(u[4 * q + 3]));
      return true;
    };
    int gq = 0;
    int n_box = 0;  // staging boxes this warp has filled
    for (int k = 0; ok; ++k) {
      int item = -1;
      if (!read_item(k, item, err) || item < 0) break;
      const BwdItem w = bwd_item<kCausal>(item, n_kt, bh_count, head_group);
      const bool key_ok = w.j * 128 + r < n;
      for (int it = 0; it < w.n_it; ++it) {
        const int t = gq + it;
        const int i = w.i0 + it;
        const uint32_t ph = t & 1;
        if (!wait_bounded_warp(bar(L::kSFull), ph, limit_ns, abort_flag, err)) {
          ok = false;
          break;
        }
        tc_fence_after();
        // keep key r for query column c iff c >= thr: r on the causal
        // diagonal, 0 elsewhere, past every column for a key beyond N.  The
        // exponentials are taken unmasked and a half with a masked column has
        // the bf16 halves of those columns cleared afterwards (one uniform
        // branch; a per-column select in the loop, or a branch inside it,
        // measured slower: extra instructions on every tile, or a second copy
        // of the loop in the instruction cache)
        const bool diag = kCausal && (i == w.j);
        const int thr = !key_ok ? (1 << 30) : (diag ? r : 0);
        uint32_t pk[32 * kHalves];  // P^T row as bf16 pairs, kept for dS
#pragma unroll
        for (int hh = 0; hh < kHalves; ++hh) {  // halves of 64 query columns
          const int h = h0 + hh;
          uint32_t u[64];
          tmem_ld_32x32b_x32(tmem + lane_off + L::kColS + h * 64,
                             *reinterpret_cast<uint32_t(*)[32]>(&u[0]));
          tmem_ld_32x32b_x32(tmem + lane_off + L::kColS + h * 64 + 32,
                             *reinterpret_cast<uint32_t(*)[32]>(&u[32]));
          tmem_wait_ld_regs(u);
#pragma unroll
          for (int e = 0; e < 64; e += 2)
            pk[hh * 32 + e / 2] = pack_bf16x2(ex2_approx(__uint_as_float(u[e]) * c_exp),
                                              ex2_approx(__uint_as_float(u[e + 1]) * c_exp));
          if (thr > h * 64) {  // some column of this half is masked
#pragma unroll
            for (int e = 0; e < 64; e += 2) {
              const int c = h * 64 + e;
              pk[hh * 32 + e / 2] &= (c >= thr ? 0x0000FFFFu : 0u) | (c + 1 >= thr ? 0xFFFF0000u : 0u);
            }
          }
          // P^T of this half over the first 32 of its own 64 TMEM columns of
          // S'^T (bf16 pairs), which have been read
          tmem_st_32x32b_x32(tmem + lane_off + L::kColS + h * 64,
                             *reinterpret_cast<const uint32_t(*)[32]>(&pk[hh * 32]));
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(L::kPReady));
        // dQ of the previous Q tile, while this tile's dV and the previous
        // tile's dK run on the tensor core (the next dQ MMA waits for this
        // tile's dS, which these warps form after the read-out)
        if (kSplitDq && it > 0 && !dq_out(t - 1, i - 1, w.bh)) {
          ok = false;
          break;
        }

        // with dQ, dS^T goes to shared memory (dK and dQ read it there) once the
        // previous tile's MMAs are done with it; without dQ it goes over the
        // dP'^T columns just read, as bf16 pairs, and dK reads it from TMEM
        if ((kDq && !wait_bounded_warp(bar(L::kDsFree), ph ^ 1, limit_ns, abort_flag, err)) ||
            !wait_bounded_warp(bar(L::kDpFull), ph, limit_ns, abort_flag, err)) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int cl = 0; cl < 2 * kHalves; ++cl) {  // 32 query columns at a time
          const int cc = 2 * h0 + cl;
          uint32_t u[32];
          tmem_ld_32x32b_x32(tmem + lane_off + L::kColDP + cc * 32, u);
          tmem_wait_ld_regs(u);
          uint32_t wv[16];
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            const uint32_t pp = pk[(cl * 32 + e) / 2];
            wv[e / 2] = pack_bf16x2(bf16_lo(pp) * __uint_as_float(u[e]),
                                    bf16_hi(pp) * __uint_as_float(u[e + 1]));
          }
          if (kDq) {
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const int qq = cc * 4 + q;  // 16-byte chunk index within the 256-byte row
              st_shared_v4(dsrow + (qq >> 3) * 16384 + (((qq & 7) ^ (r & 7)) << 4), wv[4 * q],
                           wv[4 * q + 1], wv[4 * q + 2], wv[4 * q + 3]);
            }
          } else {
            // packed columns h*64 + 16 cl .. +15, all already read (h = h0)
            tmem_st_32x32b_x16(tmem + lane_off + L::kColDP + h0 * 64 + cl * 16,
                               *reinterpret_cast<const uint32_t(*)[16]>(wv));
          }
        }
        if (!kDq) tmem_wait_st();
        tc_fence_before();
        if (kDq) fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(L::kDsReady));
      }
      if (!ok) break;
      if (kSplitDq && !dq_out(gq + w.n_it - 1, w.i0 + w.n_it - 1, w.bh)) {
        ok = false;
        break;
      }
      gq += w.n_it;
      // ----------------------------------------------------- dK, dV epilogue
      // Once the item's MMAs are done: per 32 columns each thread converts
      // its key row to bf16 (dK scaled) into one of the warp's staging boxes
      // (64-byte swizzle: 16-byte chunk q of row r at chunk q ^ ((r >> 1) & 3),
      // so the 8 rows of a shared-memory wavefront hit distinct banks) and
      // one lane stores the 32 x 32 box with TMA (rows >= N clipped).  A box's
      // earlier store must have finished reading it first.  The next item's
      // first scores are computed meanwhile.
      if (!wait_bounded_warp(bar(L::kDkdvDone), k & 1, limit_ns, abort_flag,
                             err_k | kErrRoleEpilogue)) {
        ok = false;
        break;
      }
      tc_fence_after();
      constexpr int kCols = D / 32 / (kEight ? 2 : 1);  // 32-column boxes per matrix
      const int c_first = kEight ? h0 * kCols : 0;
      const int row0 = w.j * 128 + (warp & 3) * 32;  // first key row of this warp's boxes
      // (loops kept rolled: this code runs once per item, and unrolled it
      // would crowd the hot loops out of the instruction cache)
#pragma unroll 1
      for (int which = 0; which < 2; ++which) {
        const uint32_t col = which == 0 ? L::kColDK : L::kColDV;
        const float mul = which == 0 ? scale : 1.0f;
        const CUtensorMap* map = which == 0 ? &tm_dk : &tm_dv;
#pragma unroll 1
        for (int cl = 0; cl < kCols; ++cl) {
          const int c = c_first + cl;
          uint32_t u[32];
          tmem_ld_32x32b_x32(tmem + lane_off + col + c * 32, u);
          tmem_wait_ld_regs(u);
          const uint32_t buf = box0 + static_cast<uint32_t>((n_box % kBoxes) * L::kBox);
          if (lane == 0) {
            if (kBoxes == 2)
              bulk_wait_group_read_1();
            else
              bulk_wait_group_read_0();
          }
          __syncwarp();
#pragma unroll
          for (int q = 0; q < 4; ++q)
            st_shared_v4(buf + lane * 64 + ((q ^ ((lane >> 1) & 3)) << 4),
                         pack_bf16x2(__uint_as_float(u[8 * q + 0]) * mul,
                                     __uint_as_float(u[8 * q + 1]) * mul),
                         pack_bf16x2(__uint_as_float(u[8 * q + 2]) * mul,
                                     __uint_as_float(u[8 * q + 3]) * mul),
                         pack_bf16x2(__uint_as_float(u[8 * q + 4]) * mul,
                                     __uint_as_float(u[8 * q + 5]) * mul),
                         pack_bf16x2(__uint_as_float(u[8 * q + 6]) * mul,
                                     __uint_as_float(u[8 * q + 7]) * mul));
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            if (row0 < n) tma_store_3d(map, buf, c * 32, row0, w.bh);
            bulk_commit_group();
          }
          ++n_box;
        }
      }
      // dK and dV have left TMEM: the next item may overwrite them
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(L::kDkdvFree));
    }
    // the staging boxes must be read out before the CTA's shared memory goes
    if (lane == 0) bulk_wait_group_read_0();
  } else if (kDq && !kSplitDq && warp >= 8) {
    // --------------------------------------------------------- dQ read-out
    const int c = threadIdx.x - 256;  // query row in the tile == TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t err = err_k | kErrRoleDq;
    int gq = 0;
    bool ok = true;
    for (int k = 0; ok; ++k) {
      int item = -1;
      if (!read_item(k, item, err) || item < 0) break;
      const BwdItem w = bwd_item<kCausal>(item, n_kt, bh_count, head_group);
      for (int it = 0; it < w.n_it; ++it) {
        const int t = gq + it;
        const int i = w.i0 + it;
        if (!wait_bounded_warp(bar(L::kDqFull), t & 1, limit_ns, abort_flag, err)) {
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t u[D];
#pragma unroll
        for (int cc = 0; cc < D / 32; ++cc)
          tmem_ld_32x32b_x32(tmem + lane_off + L::kColDQ + cc * 32,
                             *reinterpret_cast<uint32_t(*)[32]>(&u[cc * 32]));
        tmem_wait_ld_regs(u);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(L::kDqFree));
        // accumulator tile layout [column group of 4][128 rows][4]: lane c's four
        // columns sit next to lane c+1's, so one warp-wide vector add covers 512
        // contiguous bytes (full sectors)
        if (!dbg_check(static_cast<size_t>(w.bh) * n_kt + i <
                           static_cast<size_t>(bh_count) * n_kt,
                       err, abort_flag)) {
          ok = false;
          break;
        }
        float* dst = dq_acc + (static_cast<size_t>(w.bh) * n_kt + static_cast<size_t>(i)) * 128 * D +
                     static_cast<size_t>(c) * 4;
#pragma unroll
        for (int q = 0; q < D / 4; ++q) {
          red_add_v4(dst + q * 512, __uint_as_float(u[4 * q]), __uint_as_float(u[4 * q + 1]),
                     __uint_as_float(u[4 * q + 2]), __uint_as_float(u[4 * q + 3]));
          if (D == 128 && (q & 1)) __nanosleep(kAddGapNs);
        }
      }
      gq += w.n_it;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, L::kTmemCols);
  }
  if (threadIdx.x == 0) sched_finish(sched_slot);
}

}  // namespace fa
