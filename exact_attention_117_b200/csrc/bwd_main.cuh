// bwd_main.cuh -- main backward kernel: one CTA per (batch*head, 128-key tile).
//
// K_j and V_j stay in shared memory for the whole CTA; the Q tiles i that see
// key tile j (all of them, or i >= j under the causal mask, since Br = Bc)
// stream through.  Per Q tile, with keys on the TMEM lanes (M = 128 keys):
//
//   S^T  = K_j Q_i^T            tcgen05, A = K_j (K-major), B = Q_i (K-major)
//   dP^T = V_j dO_i^T           tcgen05, A = V_j (K-major), B = dO_i (K-major)
//   P^T  = 2^(S^T*scale*log2e - LSE2_i)   one thread per key row, masked
//   dS^T = P^T o (dP^T - D_i)
//   dV_j += P^T dO_i            tcgen05, A = P^T (smem, K-major), B = dO_i (MN-major)
//   dK_j += dS^T Q_i            tcgen05, A = dS^T (smem, K-major), B = Q_i (MN-major)
//   dQ_i  = dS K_j              tcgen05, A = dS^T read MN-major, B = K_j (MN-major)
//
// dK_j and dV_j accumulate in TMEM and are written once by this CTA (no
// atomics); dQ_i partial products are read out of TMEM by a separate warp
// group and added into the fp32 accumulator with vector atomic adds.
//
// Warp roles (384 threads): warp 0 TMA producer; warp 1 TMEM allocator and MMA
// issuer; warps 4-7 compute P^T / dS^T (thread = key row) and write dK, dV;
// warps 8-11 read dQ out of TMEM (thread = query row) and add it to global.
//
// TMEM columns:  d=128: dK [0,128) dV [128,256) S^T [256,384) dP^T [384,512),
//                       dQ reuses the dP^T columns once dS^T has been formed.
//                d=64 : dK [0,64) dV [64,128) S^T [128,256) dP^T [256,384)
//                       dQ [384,448).
#pragma once

namespace fa {

template <int D>
struct BwdLayout {
  static constexpr int kThreads = 384;
  static constexpr int kTile = 128 * D * 2;   // bytes of a K, V, Q or dO tile
  static constexpr int kSq = 128 * 128 * 2;   // bytes of the bf16 P^T or dS^T tile
  static constexpr int kOffK = 0;
  static constexpr int kOffV = kOffK + kTile;
  static constexpr int kOffQ = kOffV + kTile;
  static constexpr int kOffDO = kOffQ + kTile;
  static constexpr int kOffP = kOffDO + kTile;
  static constexpr int kOffDS = kOffP + kSq;
  static constexpr int kOffLse = kOffDS + kSq;  // 128 fp32 LSE (log2 units) of Q tile i
  static constexpr int kOffDv = kOffLse + 512;  // 128 fp32 D_i
  static constexpr int kOffBar = kOffDv + 512;
  static constexpr int kBarArea = 256;
  static constexpr int kBytes = kOffBar + kBarArea;
  static constexpr int kSmemAlloc = kBytes + 1024;
  // barriers
  static constexpr int kKvFull = 0, kQdoFull = 1, kQdoEmpty = 2, kSFull = 3, kSFree = 4,
                       kDpFull = 5, kPReady = 6, kDsReady = 7, kPdsFree = 8, kDqFull = 9,
                       kDqFree = 10, kDkdvDone = 11, kDrain = 12, kNumBars = 13;
  static constexpr int kOffSlot = kOffBar + 8 * kNumBars;
  static constexpr int kOffAbort = kOffSlot + 4;
  static_assert(kOffAbort + 4 <= kOffBar + kBarArea, "barrier area too small");
  // TMEM columns
  static constexpr uint32_t kTmemCols = 512;
  static constexpr bool kDqAliasesDp = (D == 128);
  static constexpr uint32_t kColDK = 0;
  static constexpr uint32_t kColDV = D;
  static constexpr uint32_t kColS = 2 * D;
  static constexpr uint32_t kColDP = 2 * D + 128;
  static constexpr uint32_t kColDQ = kDqAliasesDp ? kColDP : (2 * D + 256);
  static_assert(kColDQ + D <= kTmemCols, "TMEM budget");
};

template <int D, bool kCausal>
__global__ void __launch_bounds__(384, 1)
    bwd_main_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                    const float* __restrict__ dvec, const float* __restrict__ lse2,
                    float* __restrict__ dq_acc, __nv_bfloat16* __restrict__ dk,
                    __nv_bfloat16* __restrict__ dv, int n, int np, float scale, float scale_log2,
                    uint64_t limit_ns) {
  using L = BwdLayout<D>;
  constexpr int kDBlk = D / 64;

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
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
      if (b == L::kSFree || b == L::kPReady || b == L::kDsReady || b == L::kDqFree) cnt = 4;
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
        if (!wait_bounded(bar(L::kQdoEmpty), (it & 1) ^ 1, limit_ns, abort_flag,
                          err_k | kErrRoleLoad))
          break;
        mbar_arrive_expect_tx(bar(L::kQdoFull), 2 * L::kTile + 1024);
        for (int db = 0; db < kDBlk; ++db) {
          tma_load_3d(sb + L::kOffQ + db * 16384, &tm_q, bar(L::kQdoFull), db * 64, i * 128, bh);
          tma_load_3d(sb + L::kOffDO + db * 16384, &tm_do, bar(L::kQdoFull), db * 64, i * 128,
                      bh);
        }
        const size_t vrow = static_cast<size_t>(bh) * np + static_cast<size_t>(i) * 128;
        bulk_load(sb + L::kOffLse, lse2 + vrow, 512, bar(L::kQdoFull));
        bulk_load(sb + L::kOffDv, dvec + vrow, 512, bar(L::kQdoFull));
        issued = it + 1;
      }
      if (*abort_flag) {
        drain_wait(bar(L::kKvFull), 0, limit_ns);
        if (issued > 0) drain_wait(bar(L::kQdoFull), (issued - 1) & 1, limit_ns);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t id_kk = idesc_bf16_f32(128, 128, false, false);
      constexpr uint32_t id_kmn = idesc_bf16_f32(128, D, false, true);
      constexpr uint32_t id_mnmn = idesc_bf16_f32(128, D, true, true);
      const uint32_t err = err_k | kErrRoleMma;
      const uint32_t a_k = sb + L::kOffK, a_v = sb + L::kOffV, a_q = sb + L::kOffQ,
                     a_do = sb + L::kOffDO, a_p = sb + L::kOffP, a_ds = sb + L::kOffDS;
      bool ok = wait_bounded(bar(L::kKvFull), 0, limit_ns, abort_flag, err);
      for (int it = 0; ok && it < n_it; ++it) {
        const uint32_t ph = it & 1;
        if (!wait_bounded(bar(L::kQdoFull), ph, limit_ns, abort_flag, err)) break;
        if (!wait_bounded(bar(L::kSFree), ph ^ 1, limit_ns, abort_flag, err)) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {  // S^T = K_j Q_i^T
          const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
          mma_bf16_ss(tmem + L::kColS, sw128_desc(a_k + off, 16, 1024),
                      sw128_desc(a_q + off, 16, 1024), id_kk, kk > 0 ? 1u : 0u);
        }
        tc_commit(bar(L::kSFull));
        if (L::kDqAliasesDp) {
          if (!wait_bounded(bar(L::kDqFree), ph ^ 1, limit_ns, abort_flag, err)) break;
          tc_fence_after();
        }
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {  // dP^T = V_j dO_i^T
          const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
          mma_bf16_ss(tmem + L::kColDP, sw128_desc(a_v + off, 16, 1024),
                      sw128_desc(a_do + off, 16, 1024), id_kk, kk > 0 ? 1u : 0u);
        }
        tc_commit(bar(L::kDpFull));
        if (!wait_bounded(bar(L::kPReady), ph, limit_ns, abort_flag, err)) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {  // dV_j += P^T dO_i  (K = 128 queries)
          const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
          mma_bf16_ss(tmem + L::kColDV, sw128_desc(a_p + off, 16, 1024),
                      sw128_desc(a_do + kk * 2048, 16384, 1024), id_kmn,
                      (it > 0 || kk > 0) ? 1u : 0u);
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
        tc_commit(bar(L::kQdoEmpty));  // Q_i, dO_i, LSE_i, D_i no longer read
        if (!L::kDqAliasesDp) {
          if (!wait_bounded(bar(L::kDqFree), ph ^ 1, limit_ns, abort_flag, err)) break;
          tc_fence_after();
        }
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {  // dQ_i = dS K_j  (K = 128 keys)
          mma_bf16_ss(tmem + L::kColDQ, sw128_desc(a_ds + kk * 2048, 16384, 1024),
                      sw128_desc(a_k + kk * 2048, 16384, 1024), id_mnmn, kk > 0 ? 1u : 0u);
        }
        tc_commit(bar(L::kDqFull));
        tc_commit(bar(L::kPdsFree));
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
    const float4* lse4 = reinterpret_cast<const float4*>(smem + L::kOffLse);
    const float4* d4 = reinterpret_cast<const float4*>(smem + L::kOffDv);
    const uint32_t prow = sb + L::kOffP + r * 128;
    const uint32_t dsrow = sb + L::kOffDS + r * 128;
    bool ok = true;
    for (int it = 0; it < n_it; ++it) {
      const int i = i0 + it;
      const uint32_t ph = it & 1;
      if (!wait_bounded(bar(L::kQdoFull), ph, limit_ns, abort_flag, err) ||
          !wait_bounded(bar(L::kSFull), ph, limit_ns, abort_flag, err)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const bool diag = kCausal && (i == j);
      uint32_t pk[64];
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
          float p0 = ex2_approx(__uint_as_float(u[c4 * 4 + 0]) * scale_log2 - l.x);
          float p1 = ex2_approx(__uint_as_float(u[c4 * 4 + 1]) * scale_log2 - l.y);
          float p2 = ex2_approx(__uint_as_float(u[c4 * 4 + 2]) * scale_log2 - l.z);
          float p3 = ex2_approx(__uint_as_float(u[c4 * 4 + 3]) * scale_log2 - l.w);
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
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(L::kSFree));
      // the previous tile's MMAs must be done reading P^T and dS^T
      if (!wait_bounded(bar(L::kPdsFree), ph ^ 1, limit_ns, abort_flag, err)) {
        ok = false;
        break;
      }
#pragma unroll
      for (int q = 0; q < 16; ++q)
        st_shared_v4(prow + (q >> 3) * 16384 + (((q & 7) ^ (r & 7)) << 4), pk[4 * q],
                     pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(L::kPReady));

      if (!wait_bounded(bar(L::kDpFull), ph, limit_ns, abort_flag, err)) {
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
    if (ok) ok = wait_bounded(bar(L::kDkdvDone), 0, limit_ns, abort_flag, err_k | kErrRoleEpilogue);
    if (ok) {
      tc_fence_after();
      const size_t grow = (static_cast<size_t>(bh) * n + static_cast<size_t>(key)) * D;
#pragma unroll
      for (int which = 0; which < 2; ++which) {
        const uint32_t col = which == 0 ? L::kColDK : L::kColDV;
        const float mul = which == 0 ? scale : 1.0f;
        __nv_bfloat16* dst = (which == 0 ? dk : dv) + grow;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t u[32];
          tmem_ld_32x32b_x32(tmem + lane_off + col + c * 32, u);
          tmem_wait_ld();
          if (key_ok) {
#pragma unroll
            for (int q = 0; q < 4; ++q)
              st_global_v4(dst + c * 32 + q * 8,
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
      }
    }
  } else if (warp >= 8) {
    // --------------------------------------------------------- dQ read-out
    const int c = threadIdx.x - 256;  // query row in the tile == TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t err = err_k | kErrRoleDq;
    for (int it = 0; it < n_it; ++it) {
      const int i = i0 + it;
      if (!wait_bounded(bar(L::kDqFull), it & 1, limit_ns, abort_flag, err)) break;
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
      float* dst = dq_acc + (static_cast<size_t>(bh) * np + static_cast<size_t>(i) * 128 + c) * D;
#pragma unroll
      for (int q = 0; q < D / 4; ++q)
        red_add_v4(dst + 4 * q, __uint_as_float(u[4 * q]), __uint_as_float(u[4 * q + 1]),
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
