// dq_pass.cuh -- dQ without atomics: one CTA per (batch*head, 128-row Q tile).
//
// The deterministic backward splits the work of the page's recompute
// backward ("从零实现 FlashAttention-2：分块在线 Softmax", section
// 反向传播：重算，而不是存储) in two passes: the key-tile-owned main kernel
// produces dK and dV (no dQ), and this Q-tile-owned pass recomputes, for every
// key tile j the Q tile sees,
//
//   S  = Q_i K_j^T,  P = 2^(c S - LSE2_q)   (c = scale * log2 e)
//   dP = dO_i V_j^T, dS = P o (dP - D_q)
//   dQ_i += dS K_j
//
// with dQ_i accumulated in TMEM over j and written once (times the scale):
// the sum runs in one fixed order, so dQ is bitwise reproducible.  Queries
// sit on the TMEM lanes, so LSE2_q and D_q are per-thread scalars.
//
// Warp roles (384 threads): warp 0 TMA producer (Q_i and dO_i once, then
// K_j / V_j rings of three and two stages); warp 1 TMEM allocator and MMA issuer; warps 4-7
// and 8-11 two compute warpgroups, one thread per query row, the first on keys
// 0-63 of each tile, the second on keys 64-127.  TMEM: two score regions
// (S_j in region j & 1; dS_j written over its own S_j columns as bf16 pairs),
// one dP region and the dQ accumulator.  Issue order S_0, dP_0, then per key
// tile j: S_{j+1}, [dS_j ready], dQ_j, dP_{j+1} -- the next score tile is
// computed while the compute warps still work on this one, and tcgen05.mma
// ops of one thread run in issue order, so S_{j+1} only overwrites dS_{j-1}
// after dQ_{j-1} has read it.
#pragma once

#include "common.cuh"

namespace fa {

template <int D>
struct DqLayout {
  static constexpr int kThreads = 384;
  // K_j lives from S_j (issued one key tile ahead) to dQ_j, V_j only for
  // dP_j: K gets the deeper ring so that its load starts well ahead of use
  static constexpr int kKStages = 3;
  static constexpr int kVStages = 2;
  static constexpr int kTile = 128 * D * 2;
  static constexpr int kOffQ = 0;
  static constexpr int kOffDO = kTile;
  static constexpr int kOffK = 2 * kTile;
  static constexpr int kOffV = kOffK + kKStages * kTile;
  static constexpr int kOffBar = kOffV + kVStages * kTile;
  static constexpr int kBarArea = 256;
  static constexpr int kBytes = kOffBar + kBarArea;
  static constexpr int kSmemAlloc = kBytes + 1024;
  static_assert(kSmemAlloc <= 232448, "shared memory budget");
  static constexpr int kQFull = 0, kKFull = 1 /*[3]*/, kKEmpty = 4 /*[3]*/, kVFull = 7 /*[2]*/,
                       kVEmpty = 9 /*[2]*/, kSFull = 11 /*[2]*/, kDpFull = 13, kDsReady = 14,
                       kDqDone = 15, kDrain = 16, kNumBars = 17;
  static constexpr int kOffSlot = kOffBar + 8 * kNumBars;
  static constexpr int kOffAbort = kOffSlot + 4;
  static_assert(kOffAbort + 4 <= kOffBar + kBarArea, "barrier area too small");
  static constexpr uint32_t kTmemCols = 512;
  // score region of key tile j starts at column 128 * (j & 1)
  static __device__ __forceinline__ uint32_t col_s(int j) { return static_cast<uint32_t>(j & 1) * 128u; }
  static constexpr uint32_t kColDP = 256;
  static constexpr uint32_t kColDQ = 384;
  static_assert(kColDQ + D <= kTmemCols, "TMEM budget");
};

template <int D, bool kCausal>
__global__ void __launch_bounds__(384, 1)
    dq_pass_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                   const __grid_constant__ CUtensorMap tm_dq, const float* __restrict__ dvec,
                   const float* __restrict__ lse2, int n, int np, float scale, float c_exp,
                   uint64_t limit_ns, int bh_count, int head_group) {
  using L = DqLayout<D>;
  constexpr int KS = L::kKStages;
  constexpr int VS = L::kVStages;
  constexpr int kDBlk = D / 64;

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
  const uint32_t sb = smem_u32(smem);
  auto bar = [&](int b) -> uint32_t { return sb + L::kOffBar + 8u * static_cast<uint32_t>(b); };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kOffAbort);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kOffSlot);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // Launch order: heads in groups of head_group, and within a group the
  // longest causal rows first (Q tile n-1 of every head of the group, then
  // n-2, ...), so the CTAs in flight share the K and V tiles of a few heads
  // in L2.
  const int n_tiles = np / 128;
  const int lin = static_cast<int>(blockIdx.x);
  const int grp = lin / (head_group * n_tiles);
  const int g_base = grp * head_group;
  const int g_size = min(head_group, bh_count - g_base);
  const int g_off = lin - grp * head_group * n_tiles;
  const int bh = g_base + g_off % g_size;
  const int i = n_tiles - 1 - g_off / g_size;
  const int n_kv = kCausal ? i + 1 : n_tiles;
  const unsigned int err_k = kErrBwdDq;

  if (threadIdx.x == 0) {
    for (int b = 0; b < L::kNumBars; ++b) mbar_init(bar(b), b == L::kDsReady ? 8u : 1u);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), L::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      tma_prefetch_desc(&tm_do);
      const uint32_t err = err_k | kErrRoleLoad;
      // a failed check raises the abort flag; the other roles then give up
      const bool q_ok = dbg_check(i * 128 < n && n_kv * 128 <= np, err, abort_flag);
      if (q_ok) {
        mbar_arrive_expect_tx(bar(L::kQFull), 2 * L::kTile);
        for (int db = 0; db < kDBlk; ++db) {
          tma_load_3d(sb + L::kOffQ + db * 16384, &tm_q, bar(L::kQFull), db * 64, i * 128, bh);
          tma_load_3d(sb + L::kOffDO + db * 16384, &tm_do, bar(L::kQFull), db * 64, i * 128, bh);
        }
      }
      int nk = 0, nv = 0;
      for (int j = 0; q_ok && j < n_kv; ++j) {
        const int sk = j % KS, sv = j % VS;
        if (!dbg_check(j * 128 < n, err, abort_flag) ||
            !wait_bounded(bar(L::kKEmpty + sk), ((j / KS) & 1) ^ 1, limit_ns, abort_flag, err))
          break;
        mbar_arrive_expect_tx(bar(L::kKFull + sk), L::kTile);
        for (int db = 0; db < kDBlk; ++db)
          tma_load_3d(sb + L::kOffK + sk * L::kTile + db * 16384, &tm_k, bar(L::kKFull + sk),
                      db * 64, j * 128, bh);
        ++nk;
        if (!wait_bounded(bar(L::kVEmpty + sv), ((j / VS) & 1) ^ 1, limit_ns, abort_flag, err))
          break;
        mbar_arrive_expect_tx(bar(L::kVFull + sv), L::kTile);
        for (int db = 0; db < kDBlk; ++db)
          tma_load_3d(sb + L::kOffV + sv * L::kTile + db * 16384, &tm_v, bar(L::kVFull + sv),
                      db * 64, j * 128, bh);
        ++nv;
      }
      if (*abort_flag && q_ok) {
        drain_wait(bar(L::kQFull), 0, limit_ns);
        for (int j = (nk > KS ? nk - KS : 0); j < nk; ++j)
          drain_wait(bar(L::kKFull + j % KS), (j / KS) & 1, limit_ns);
        for (int j = (nv > VS ? nv - VS : 0); j < nv; ++j)
          drain_wait(bar(L::kVFull + j % VS), (j / VS) & 1, limit_ns);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // the whole warp runs this loop; the MMA and commit wrappers elect one lane
    {
      constexpr uint32_t id_kk = idesc_bf16_f32(128, 128, false, false);
      constexpr uint32_t id_kmn = idesc_bf16_f32(128, D, false, true);
      const uint32_t err = err_k | kErrRoleMma;
      const uint32_t a_q = sb + L::kOffQ, a_do = sb + L::kOffDO;
      auto issue_s = [&](int j) {  // S_j = Q_i K_j^T into score region j & 1
        const uint32_t b_k = sb + L::kOffK + (j % KS) * L::kTile;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
          mma_bf16_ss(tmem + L::col_s(j), sw128_desc(a_q + off, 16, 1024),
                      sw128_desc(b_k + off, 16, 1024), id_kk, kk > 0 ? 1u : 0u);
        }
        tc_commit(bar(L::kSFull + (j & 1)));
      };
      auto issue_dp = [&](int j) {  // dP_j = dO_i V_j^T
        const uint32_t b_v = sb + L::kOffV + (j % VS) * L::kTile;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
          mma_bf16_ss(tmem + L::kColDP, sw128_desc(a_do + off, 16, 1024),
                      sw128_desc(b_v + off, 16, 1024), id_kk, kk > 0 ? 1u : 0u);
        }
        tc_commit(bar(L::kDpFull));
        tc_commit(bar(L::kVEmpty + (j % VS)));  // V_j is read only by dP_j
      };
      bool ok = wait_bounded_warp(bar(L::kQFull), 0, limit_ns, abort_flag, err) &&
                wait_bounded_warp(bar(L::kKFull), 0, limit_ns, abort_flag, err) &&
                wait_bounded_warp(bar(L::kVFull), 0, limit_ns, abort_flag, err);
      if (ok) {
        tc_fence_after();
        issue_s(0);
        issue_dp(0);
      }
      for (int j = 0; ok && j < n_kv; ++j) {
        const int s = j % KS;
        const bool next = j + 1 < n_kv;
        if (next) {  // S_{j+1} into the region dQ_{j-1} has finished reading
          if (!wait_bounded_warp(bar(L::kKFull + (j + 1) % KS), ((j + 1) / KS) & 1, limit_ns,
                            abort_flag, err))
            break;
          tc_fence_after();
          issue_s(j + 1);
        }
        if (!wait_bounded_warp(bar(L::kDsReady), j & 1, limit_ns, abort_flag, err)) break;
        tc_fence_after();
        // dQ_i += dS_j K_j: A = dS_j from TMEM (keys 0-63 at columns 0-31 of
        // the region, keys 64-127 at columns 64-95), B = K_j MN-major
        const uint32_t b_k = sb + L::kOffK + s * L::kTile;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_bf16_ts(tmem + L::kColDQ, tmem + L::col_s(j) + (kk >> 2) * 64 + (kk & 3) * 8,
                      sw128_desc(b_k + kk * 2048, 16384, 1024), id_kmn,
                      (j > 0 || kk > 0) ? 1u : 0u);
        tc_commit(bar(L::kKEmpty + s));  // K_j: read by S_j and this dQ step
        if (next) {  // dP_{j+1}: the compute warps have read dP_j
          if (!wait_bounded_warp(bar(L::kVFull + (j + 1) % VS), ((j + 1) / VS) & 1, limit_ns,
                            abort_flag, err))
            break;
          tc_fence_after();
          issue_dp(j + 1);
        }
      }
      tc_commit(bar(L::kDqDone));
      tc_commit(bar(L::kDrain));
      drain_wait(bar(L::kDrain), 0, limit_ns);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ----------------------------------------- P, dS (thread = query row)
    const int wg = (warp >> 2) - 1;  // 0: keys 0-63, 1: keys 64-127
    const int r = (warp & 3) * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t cb = static_cast<uint32_t>(wg) * 64u;
    const uint32_t err = err_k | kErrRoleSoftmax;
    const int q = i * 128 + r;  // query row
    const size_t vrow = static_cast<size_t>(bh) * np + q;
    const float l2 = lse2[vrow];
    const float dd = dvec[vrow];
    // rows past the end (LSE2 = +inf) get probability 0 everywhere
    const float neg_l2 = (l2 == INFINITY) ? -INFINITY : -l2;
    bool ok = true;
    for (int j = 0; j < n_kv; ++j) {
      const uint32_t xa = tmem + lane_off + L::col_s(j) + cb;  // S_j, then dS_j
      if (!wait_bounded_warp(bar(L::kSFull + (j & 1)), (j >> 1) & 1, limit_ns, abort_flag, err)) {
        ok = false;
        break;
      }
      tc_fence_after();
      // keys of this tile that row q sees: k <= q (causal), k < n
      int lim = 128;
      if (kCausal && j == i) lim = r + 1;
      const int rem = n - j * 128;
      if (rem < lim) lim = rem;
      lim -= static_cast<int>(cb);
      uint32_t pk[32];
      {
        uint32_t u[64];
        tmem_ld_32x32b_x32(xa, *reinterpret_cast<uint32_t(*)[32]>(&u[0]));
        tmem_ld_32x32b_x32(xa + 32, *reinterpret_cast<uint32_t(*)[32]>(&u[32]));
        tmem_wait_ld_regs(u);
#pragma unroll
        for (int e = 0; e < 64; e += 2) {
          float p0 = ex2_approx(fmaf(__uint_as_float(u[e]), c_exp, neg_l2));
          float p1 = ex2_approx(fmaf(__uint_as_float(u[e + 1]), c_exp, neg_l2));
          p0 = (e < lim) ? p0 : 0.f;
          p1 = (e + 1 < lim) ? p1 : 0.f;
          pk[e / 2] = pack_bf16x2(p0, p1);
        }
      }
      if (!wait_bounded_warp(bar(L::kDpFull), j & 1, limit_ns, abort_flag, err)) {
        ok = false;
        break;
      }
      tc_fence_after();
      {
        uint32_t u[64];
        const uint32_t ya = tmem + lane_off + L::kColDP + cb;
        tmem_ld_32x32b_x32(ya, *reinterpret_cast<uint32_t(*)[32]>(&u[0]));
        tmem_ld_32x32b_x32(ya + 32, *reinterpret_cast<uint32_t(*)[32]>(&u[32]));
        tmem_wait_ld_regs(u);
        uint32_t w[32];
#pragma unroll
        for (int e = 0; e < 64; e += 2) {
          const uint32_t pp = pk[e / 2];
          w[e / 2] = pack_bf16x2(bf16_lo(pp) * (__uint_as_float(u[e]) - dd),
                                 bf16_hi(pp) * (__uint_as_float(u[e + 1]) - dd));
        }
        // dS over this warpgroup's own S_j columns, which it has read
        tmem_st_32x32b_x32(xa, w);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(L::kDsReady));
    }
    // -------------------------------------------------------- dQ epilogue
    // each warpgroup converts half of dQ's D columns
    if (ok) ok = wait_bounded_warp(bar(L::kDqDone), 0, limit_ns, abort_flag, err_k | kErrRoleEpilogue);
    if (ok) {
      tc_fence_after();
      const uint32_t orow = sb + L::kOffQ + r * 128;  // Q_i is dead: stage dQ there
#pragma unroll
      for (int c = 0; c < D / 64; ++c) {
        const int c0 = wg * (D / 2) + c * 32;  // first dQ column of this load
        uint32_t u[32];
        tmem_ld_32x32b_x32(tmem + lane_off + L::kColDQ + c0, u);
        tmem_wait_ld_regs(u);
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          const int jj = c0 / 8 + g;  // 16-byte chunk of the output row
          st_shared_v4(orow + (jj >> 3) * 16384 + (((jj & 7) ^ (r & 7)) << 4),
                       pack_bf16x2(__uint_as_float(u[8 * g + 0]) * scale,
                                   __uint_as_float(u[8 * g + 1]) * scale),
                       pack_bf16x2(__uint_as_float(u[8 * g + 2]) * scale,
                                   __uint_as_float(u[8 * g + 3]) * scale),
                       pack_bf16x2(__uint_as_float(u[8 * g + 4]) * scale,
                                   __uint_as_float(u[8 * g + 5]) * scale),
                       pack_bf16x2(__uint_as_float(u[8 * g + 6]) * scale,
                                   __uint_as_float(u[8 * g + 7]) * scale));
        }
      }
      fence_proxy_async_smem();
    }
    tc_fence_before();
    named_barrier_sync(1, 256);
    if (threadIdx.x == 128 && ok && !*abort_flag) {
      for (int db = 0; db < kDBlk; ++db)
        tma_store_3d(&tm_dq, sb + L::kOffQ + db * 16384, db * 64, i * 128, bh);
      bulk_commit_group();
      bulk_wait_group_read_0();
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, L::kTmemCols);
  }
}

}  // namespace fa
