// bwd_main.cuh -- main backward kernel: one CTA per (batch*head, 128-key tile).
//
// K_j and V_j stay in shared memory for the whole CTA; the Q tiles i that see
// key tile j (all of them, or i >= j under the causal mask, since Br = Bc)
// stream through a two-stage ring together with dO_i, LSE_i and D_i.  Per Q
// tile, with keys on the TMEM lanes (M = 128 keys):
//
//   S^T  = K_j Q_i^T            tcgen05, A = K_j (K-major), B = Q_i (K-major)
//   dP^T = V_j dO_i^T           tcgen05, A = V_j (K-major), B = dO_i (K-major)
//   P^T  = 2^(S^T*scale*log2e - LSE2_i)   one thread per key row, masked,
//                               written back over S^T in TMEM as bf16
//   dV_j += P^T dO_i            tcgen05, A = P^T (TMEM), B = dO_i (MN-major)
//   dS^T = P^T o (dP^T - D_i)   written to shared memory as bf16
//   dK_j += dS^T Q_i            tcgen05, A = dS^T (K-major), B = Q_i (MN-major)
//   dQ_i  = dS K_j              tcgen05, A = dS^T read MN-major, B = K_j (MN-major)
//
// Issue order of the tensor-core work: ... dV_i, S_{i+1}, dK_i, dQ_i, dP_{i+1},
// dV_{i+1} ...  S_{i+1} goes right after dV_i (tcgen05.mma ops of one thread
// run in order, so it cannot overwrite P_i before dV_i has read it), which lets
// the exponentials of tile i+1 overlap dK_i and dQ_i on the tensor core.
//
// dK_j and dV_j accumulate in TMEM and are written once by this CTA (no
// atomics), staged through shared memory and stored with TMA; dQ_i partial
// products are read out of TMEM by a separate warp group and added into the
// fp32 accumulator with vector atomic adds.  The accumulator keeps each
// 128-row tile as [D/4 column groups][128 rows][4 floats] so that those adds
// are coalesced.
//
// Warp roles (384 threads): warp 0 TMA producer; warp 1 TMEM allocator and MMA
// issuer; warps 4-7 compute P^T / dS^T (thread = key row) and write dK, dV;
// warps 8-11 read dQ out of TMEM (thread = query row) and add it to global.
//
// TMEM columns:  dK [0,D), dV [D,2D), S^T/P^T [2D,2D+128), dP^T [2D+128,2D+256);
// dQ reuses the dP^T columns once dS^T has been formed (d=128 fills all 512).
#pragma once

namespace fa {

template <int D>
struct BwdLayout {
  static constexpr int kThreads = 384;
  static constexpr int kTile = 128 * D * 2;  // bytes of a K, V, Q or dO tile
  static constexpr int kSq = 128 * 128 * 2;  // bytes of the bf16 dS^T tile
  static constexpr int kOffK = 0;
  static constexpr int kOffV = kOffK + kTile;
  static constexpr int kOffQ = kOffV + kTile;    // [2]
  static constexpr int kOffDO = kOffQ + 2 * kTile;  // [2]
  static constexpr int kOffDS = kOffDO + 2 * kTile;
  static constexpr int kOffLse = kOffDS + kSq;  // [2] x 128 fp32 LSE (log2 units) of Q tile i
  static constexpr int kOffDv = kOffLse + 1024;  // [2] x 128 fp32 D_i
  static constexpr int kOffBar = kOffDv + 1024;
  static constexpr int kBarArea = 256;
  static constexpr int kBytes = kOffBar + kBarArea;
  // The 1 KiB alignment slack is kept only where it fits; without it the
  // kernel checks that the dynamic shared memory base is 1 KiB aligned.
  static constexpr int kSlack = (kBytes + 1024 <= 232448) ? 1024 : 0;
  static constexpr int kSmemAlloc = kBytes + kSlack;
  static_assert(kSmemAlloc <= 232448, "shared memory budget");
  // barriers
  static constexpr int kKvFull = 0, kQdoFull = 1 /*[2]*/, kQdoEmpty = 3 /*[2]*/, kSFull = 5,
                       kPReady = 6, kDpFull = 7, kDsReady = 8, kDsFree = 9, kDqFull = 10,
                       kDqFree = 11, kDkdvDone = 12, kDrain = 13, kNumBars = 14;
  static constexpr int kOffSlot = kOffBar + 8 * kNumBars;
  static constexpr int kOffAbort = kOffSlot + 4;
  static_assert(kOffAbort + 4 <= kOffBar + kBarArea, "barrier area too small");
  // TMEM columns
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kColDK = 0;
  static constexpr uint32_t kColDV = D;
  static constexpr uint32_t kColS = 2 * D;
  static constexpr uint32_t kColDP = 2 * D + 128;
  static constexpr uint32_t kColDQ = kColDP;
  static_assert(kColDP + 128 <= kTmemCols, "TMEM budget");
};

template <int D, bool kCausal>
__global__ void __launch_bounds__(384, 1)
    bwd_main_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                    const __grid_constant__ CUtensorMap tm_dk, const __grid_constant__ CUtensorMap tm_dv,
                    const float* __restrict__ dvec, const float* __restrict__ lse2,
                    float* __restrict__ dq_acc, int n, int np, float scale, float scale_log2,
                    uint64_t limit_ns) {
  using L = BwdLayout<D>;
  constexpr int kDBlk = D / 64;

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  if (L::kSlack == 0 && (raw_addr & 1023u) != 0) {
    // every thread sees the same base: the whole CTA leaves before touching
    // any barrier or TMEM
    if (threadIdx.x == 0) atomicOr(&g_error_word, kErrBwdMain | kErrAlign);
    return;
  }
  uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
  const uint32_t sb = smem_u32(smem);
  auto bar = [&](int i) -> uint32_t { return sb + L::kOffBar + 8u * static_cast<uint32_t>(i); };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kOffAbort);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kOffSlot);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int bh = blockIdx.x;
  const int j = blockIdx.y;  // key tile; small j (most Q tiles under causal) first
  const int n_q = np / 128;
  const int i0 = kCausal ? j : 0;
  const int n_it = n_q - i0;
  const unsigned int err_k = kErrBwdMain;

  if (threadIdx.x == 0) {
    for (int b = 0; b < L::kNumBars; ++b) {
      uint32_t cnt = 1;
      if (b == L::kPReady || b == L::kDsReady || b == L::kDqFree) cnt = 4;
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

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      tma_prefetch_desc(&tm_do);
      mbar_arrive_expect_tx(bar(L::kKvFull), 2 * L::kTile);
      for (int db = 0; db < kDBlk; ++db) {
        tma_load_3d(sb + L::kOffK + db * 16384, &tm_k, bar(L::kKvFull), db * 64, j * 128, bh);
        tma_load_3d(sb + L::kOffV + db * 16384, &tm_v, bar(L::kKvFull), db * 64, j * 128, bh);
      }
      int issued = 0;
      for (int it = 0; it < n_it; ++it) {
        const int i = i0 + it;
        const int st = it & 1;
        if (!wait_bounded(bar(L::kQdoEmpty + st), ((it >> 1) & 1) ^ 1, limit_ns, abort_flag,
                          err_k | kErrRoleLoad))
          break;
        const uint32_t fb = bar(L::kQdoFull + st);
        mbar_arrive_expect_tx(fb, 2 * L::kTile + 1024);
        for (int db = 0; db < kDBlk; ++db) {
          tma_load_3d(sb + L::kOffQ + st * L::kTile + db * 16384, &tm_q, fb, db * 64, i * 128, bh);
          tma_load_3d(sb + L::kOffDO + st * L::kTile + db * 16384, &tm_do, fb, db * 64, i * 128,
                      bh);
        }
        const size_t vrow = static_cast<size_t>(bh) * np + static_cast<size_t>(i) * 128;
        bulk_load(sb + L::kOffLse + st * 512, lse2 + vrow, 512, fb);
        bulk_load(sb + L::kOffDv + st * 512, dvec + vrow, 512, fb);
        issued = it + 1;
      }
      if (*abort_flag) {
        drain_wait(bar(L::kKvFull), 0, limit_ns);
        for (int it = (issued > 2 ? issued - 2 : 0); it < issued; ++it)
          drain_wait(bar(L::kQdoFull + (it & 1)), (it >> 1) & 1, limit_ns);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t id_kk = idesc_bf16_f32(128, 128, false, false);
      constexpr uint32_t id_kmn = idesc_bf16_f32(128, D, false, true);
      constexpr uint32_t id_mnmn = idesc_bf16_f32(128, D, true, true);
      const uint32_t err = err_k | kErrRoleMma;
      const uint32_t a_k = sb + L::kOffK, a_v = sb + L::kOffV, a_ds = sb + L::kOffDS;
      auto issue_s = [&](int it) {  // S^T = K_j Q_i^T
        const uint32_t a_q = sb + L::kOffQ + (it & 1) * L::kTile;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
          mma_bf16_ss(tmem + L::kColS, sw128_desc(a_k + off, 16, 1024),
                      sw128_desc(a_q + off, 16, 1024), id_kk, kk > 0 ? 1u : 0u);
        }
        tc_commit(bar(L::kSFull));
      };
      auto issue_dp = [&](int it) {  // dP^T = V_j dO_i^T
        const uint32_t a_do = sb + L::kOffDO + (it & 1) * L::kTile;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
          mma_bf16_ss(tmem + L::kColDP, sw128_desc(a_v + off, 16, 1024),
                      sw128_desc(a_do + off, 16, 1024), id_kk, kk > 0 ? 1u : 0u);
        }
        tc_commit(bar(L::kDpFull));
      };
      bool ok = wait_bounded(bar(L::kKvFull), 0, limit_ns, abort_flag, err) &&
                wait_bounded(bar(L::kQdoFull), 0, limit_ns, abort_flag, err);
      if (ok) {
        tc_fence_after();
        issue_s(0);
        issue_dp(0);
      }
      for (int it = 0; ok && it < n_it; ++it) {
        const uint32_t ph = it & 1;
        const int st = it & 1;
        const uint32_t a_q = sb + L::kOffQ + st * L::kTile;
        const uint32_t a_do = sb + L::kOffDO + st * L::kTile;
        const bool next = it + 1 < n_it;
        if (!wait_bounded(bar(L::kPReady), ph, limit_ns, abort_flag, err)) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)  // dV_j += P^T dO_i  (K = 128 queries, P^T in TMEM)
          mma_bf16_ts(tmem + L::kColDV, tmem + L::kColS + kk * 8,
                      sw128_desc(a_do + kk * 2048, 16384, 1024), id_kmn,
                      (it > 0 || kk > 0) ? 1u : 0u);
        if (next) {  // S of the next Q tile, as soon as P_i has been consumed
          if (!wait_bounded(bar(L::kQdoFull + ((it + 1) & 1)), ((it + 1) >> 1) & 1, limit_ns,
                            abort_flag, err))
            break;
          tc_fence_after();
          issue_s(it + 1);
        }
        if (!wait_bounded(bar(L::kDsReady), ph, limit_ns, abort_flag, err)) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {  // dK_j += dS^T Q_i
          const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
          mma_bf16_ss(tmem + L::kColDK, sw128_desc(a_ds + off, 16, 1024),
                      sw128_desc(a_q + kk * 2048, 16384, 1024), id_kmn,
                      (it > 0 || kk > 0) ? 1u : 0u);
        }
        tc_commit(bar(L::kQdoEmpty + st));  // Q_i, dO_i, LSE_i, D_i no longer read
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)  // dQ_i = dS K_j  (K = 128 keys)
          mma_bf16_ss(tmem + L::kColDQ, sw128_desc(a_ds + kk * 2048, 16384, 1024),
                      sw128_desc(a_k + kk * 2048, 16384, 1024), id_mnmn, kk > 0 ? 1u : 0u);
        tc_commit(bar(L::kDqFull));
        tc_commit(bar(L::kDsFree));
        if (next) {  // dP of the next Q tile once dQ_i has left the shared columns
          if (!wait_bounded(bar(L::kDqFree), ph, limit_ns, abort_flag, err)) break;
          tc_fence_after();
          issue_dp(it + 1);
        }
      }
      tc_commit(bar(L::kDkdvDone));
      tc_commit(bar(L::kDrain));
      drain_wait(bar(L::kDrain), 0, limit_ns);
    }
    __syncwarp();
  } else if (warp >= 4 && warp < 8) {
    // ------------------------------------------------ P^T, dS^T, dK / dV out
    const int r = threadIdx.x - 128;  // key row in the tile == TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const int key = j * 128 + r;
    const bool key_ok = key < n;
    const uint32_t err = err_k | kErrRoleSoftmax;
    const uint32_t dsrow = sb + L::kOffDS + r * 128;
    bool ok = true;
    for (int it = 0; it < n_it; ++it) {
      const int i = i0 + it;
      const uint32_t ph = it & 1;
      const int st = it & 1;
      const float4* lse4 = reinterpret_cast<const float4*>(smem + L::kOffLse + st * 512);
      const float4* d4 = reinterpret_cast<const float4*>(smem + L::kOffDv + st * 512);
      if (!wait_bounded_warp(bar(L::kQdoFull + st), (it >> 1) & 1, limit_ns, abort_flag, err) ||
          !wait_bounded_warp(bar(L::kSFull), ph, limit_ns, abort_flag, err)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const bool diag = kCausal && (i == j);
      uint32_t pk[64];  // P^T row as bf16 pairs, kept for dS
#pragma unroll
      for (int h = 0; h < 2; ++h) {  // two halves of 64 query columns
        uint32_t u[64];
        tmem_ld_32x32b_x32(tmem + lane_off + L::kColS + h * 64,
                           *reinterpret_cast<uint32_t(*)[32]>(&u[0]));
        tmem_ld_32x32b_x32(tmem + lane_off + L::kColS + h * 64 + 32,
                           *reinterpret_cast<uint32_t(*)[32]>(&u[32]));
        tmem_wait_ld();
#pragma unroll
        for (int c4 = 0; c4 < 16; ++c4) {
          const float4 l = lse4[h * 16 + c4];
          const int c = h * 64 + c4 * 4;
          float p0 = ex2_approx(fmaf(__uint_as_float(u[c4 * 4 + 0]), scale_log2, -l.x));
          float p1 = ex2_approx(fmaf(__uint_as_float(u[c4 * 4 + 1]), scale_log2, -l.y));
          float p2 = ex2_approx(fmaf(__uint_as_float(u[c4 * 4 + 2]), scale_log2, -l.z));
          float p3 = ex2_approx(fmaf(__uint_as_float(u[c4 * 4 + 3]), scale_log2, -l.w));
          if (diag) {  // keep key r for query c iff r <= c
            p0 = (c + 0 >= r) ? p0 : 0.f;
            p1 = (c + 1 >= r) ? p1 : 0.f;
            p2 = (c + 2 >= r) ? p2 : 0.f;
            p3 = (c + 3 >= r) ? p3 : 0.f;
          }
          if (!key_ok) p0 = p1 = p2 = p3 = 0.f;
          pk[c / 2] = pack_bf16x2(p0, p1);
          pk[c / 2 + 1] = pack_bf16x2(p2, p3);
        }
        // P^T over the first 64 TMEM columns of S^T (bf16 pairs): this half's
        // 32 packed columns land on S^T columns already read
        tmem_st_32x32b_x32(tmem + lane_off + L::kColS + h * 32,
                           *reinterpret_cast<const uint32_t(*)[32]>(&pk[h * 32]));
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(L::kPReady));

      // the previous tile's MMAs must be done reading dS^T
      if (!wait_bounded_warp(bar(L::kDsFree), ph ^ 1, limit_ns, abort_flag, err) ||
          !wait_bounded_warp(bar(L::kDpFull), ph, limit_ns, abort_flag, err)) {
        ok = false;
        break;
      }
      tc_fence_after();
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {  // 32 query columns at a time
        uint32_t u[32];
        tmem_ld_32x32b_x32(tmem + lane_off + L::kColDP + cc * 32, u);
        tmem_wait_ld();
        uint32_t w[16];
#pragma unroll
        for (int e = 0; e < 32; e += 4) {
          const int c = cc * 32 + e;
          const float4 dd = d4[c / 4];
          const uint32_t pa = pk[c / 2], pb = pk[c / 2 + 1];
          const float s0 = bf16_lo(pa) * (__uint_as_float(u[e + 0]) - dd.x);
          const float s1 = bf16_hi(pa) * (__uint_as_float(u[e + 1]) - dd.y);
          const float s2 = bf16_lo(pb) * (__uint_as_float(u[e + 2]) - dd.z);
          const float s3 = bf16_hi(pb) * (__uint_as_float(u[e + 3]) - dd.w);
          w[e / 2] = pack_bf16x2(s0, s1);
          w[e / 2 + 1] = pack_bf16x2(s2, s3);
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int qq = cc * 4 + q;  // 16-byte chunk index within the 256-byte row
          st_shared_v4(dsrow + (qq >> 3) * 16384 + (((qq & 7) ^ (r & 7)) << 4), w[4 * q],
                       w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
        }
      }
      tc_fence_before();
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(L::kDsReady));
    }
    // ------------------------------------------------------- dK, dV epilogue
    // dK (scaled) then dV go through the dS^T tile (free once every MMA is
    // done) as bf16 128-byte-swizzled rows, stored with TMA (rows >= N clip).
    if (ok) ok = wait_bounded_warp(bar(L::kDkdvDone), 0, limit_ns, abort_flag, err_k | kErrRoleEpilogue);
#pragma unroll
    for (int which = 0; which < 2; ++which) {
      if (ok) {
        tc_fence_after();
        const uint32_t col = which == 0 ? L::kColDK : L::kColDV;
        const float mul = which == 0 ? scale : 1.0f;
        const uint32_t orow = sb + L::kOffDS + r * 128;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t u[32];
          tmem_ld_32x32b_x32(tmem + lane_off + col + c * 32, u);
          tmem_wait_ld();
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int jj = c * 4 + q;
            st_shared_v4(orow + (jj >> 3) * 16384 + (((jj & 7) ^ (r & 7)) << 4),
                         pack_bf16x2(__uint_as_float(u[8 * q + 0]) * mul,
                                     __uint_as_float(u[8 * q + 1]) * mul),
                         pack_bf16x2(__uint_as_float(u[8 * q + 2]) * mul,
                                     __uint_as_float(u[8 * q + 3]) * mul),
                         pack_bf16x2(__uint_as_float(u[8 * q + 4]) * mul,
                                     __uint_as_float(u[8 * q + 5]) * mul),
                         pack_bf16x2(__uint_as_float(u[8 * q + 6]) * mul,
                                     __uint_as_float(u[8 * q + 7]) * mul));
          }
        }
        fence_proxy_async_smem();
      }
      tc_fence_before();
      named_barrier_sync(1, 128);  // all four warps, ok or not
      if (r == 0 && ok && !*abort_flag) {
        const CUtensorMap* map = which == 0 ? &tm_dk : &tm_dv;
        for (int db = 0; db < kDBlk; ++db)
          tma_store_3d(map, sb + L::kOffDS + db * 16384, db * 64, j * 128, bh);
        bulk_commit_group();
        bulk_wait_group_0();  // the staging tile is reused for dV
      }
      named_barrier_sync(1, 128);
    }
  } else if (warp >= 8) {
    // --------------------------------------------------------- dQ read-out
    const int c = threadIdx.x - 256;  // query row in the tile == TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t err = err_k | kErrRoleDq;
    for (int it = 0; it < n_it; ++it) {
      const int i = i0 + it;
      if (!wait_bounded_warp(bar(L::kDqFull), it & 1, limit_ns, abort_flag, err)) break;
      tc_fence_after();
      uint32_t u[D];
#pragma unroll
      for (int cc = 0; cc < D / 32; ++cc)
        tmem_ld_32x32b_x32(tmem + lane_off + L::kColDQ + cc * 32,
                           *reinterpret_cast<uint32_t(*)[32]>(&u[cc * 32]));
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(L::kDqFree));
      // accumulator tile layout [column group of 4][128 rows][4]: lane c's four
      // columns sit next to lane c+1's, so one warp-wide vector add covers 512
      // contiguous bytes (full sectors)
      float* dst = dq_acc + (static_cast<size_t>(bh) * n_q + static_cast<size_t>(i)) * 128 * D +
                   static_cast<size_t>(c) * 4;
#pragma unroll
      for (int q = 0; q < D / 4; ++q)
        red_add_v4(dst + q * 512, __uint_as_float(u[4 * q]), __uint_as_float(u[4 * q + 1]),
                   __uint_as_float(u[4 * q + 2]), __uint_as_float(u[4 * q + 3]));
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
