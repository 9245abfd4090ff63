// kv_outer.cuh -- forward attention in the FlashAttention-1 loop order, for
// measuring what that order costs on sm_100a.
//
// Page "从零实现 FlashAttention-2：分块在线 Softmax", section 从 FlashAttention-1
// 到 FlashAttention-2: the first version walks the key/value tiles in the
// OUTER loop and the query tiles in the inner loop; the second swaps them so a
// Q tile stays on chip, and also parallelises over the sequence, not only over
// batch and head.  This kernel keeps the first order on purpose:
//
//   for each key tile j (K_j, V_j loaded once):
//     for each query tile i that sees j:
//       load Q_i and the row statistics m_i, l_i and output O_i (fp32) of the
//       earlier key tiles from global memory;
//       S = Q_i K_j^T; m_new = max(m_i, rowmax S); P = 2^(S c - m_new);
//       l_new = 2^(m_i - m_new) l_i + rowsum P;
//       O_i = (2^(m_i - m_new) l_i O_i + P V_j) / l_new        (page 3 merge)
//       write m_new, l_new and O_i back (bf16 O and LSE after the last j).
//
// One CTA per (batch, head), as in that design: the query tiles of a head share
// the running O_i across key tiles, so they are not split over CTAs.  Every
// (i, j) step reads Q_i and reads and writes the fp32 O_i: the extra global
// traffic and the per-step normalisation are what the measurement shows.
//
// Warp roles (256 threads): warp 0 TMA producer (K_j / V_j in a two-stage ring,
// Q_i in a two-stage ring); warp 1 TMEM allocator and MMA issuer; warps 4-7
// softmax and O update, one thread per query row.  Step q uses TMEM score
// region q & 1 (P over its first 64 columns as bf16, the P V operand) and P V
// region q & 1.  Issue order S(q+1), P V(q): the next score tile is computed
// while the softmax warps work on this one; they update O of step q after
// forming P of step q + 1.
#pragma once

#include "common.cuh"

namespace fa {

template <int D>
struct KvOuterLayout {
  static constexpr int kTile = 128 * D * 2;
  static constexpr int kOffK = 0;                  // [2]
  static constexpr int kOffV = 2 * kTile;          // [2]
  static constexpr int kOffQ = 4 * kTile;          // [2]
  static constexpr int kOffStage = 6 * kTile;      // bf16 O staging for the TMA store
  static constexpr int kOffBar = 7 * kTile;
  static constexpr int kBarArea = 256;
  static constexpr int kBytes = kOffBar + kBarArea;
  static constexpr int kSmemAlloc = kBytes + 1024;
  static_assert(kSmemAlloc <= 232448, "shared memory budget");
  static constexpr int kKvFull = 0 /*[2]*/, kKvEmpty = 2 /*[2]*/, kQFull = 4 /*[2]*/,
                       kQEmpty = 6 /*[2]*/, kSFull = 8 /*[2]*/, kPReady = 10 /*[2]*/,
                       kPvFull = 12 /*[2]*/, kPvFree = 14 /*[2]*/, kDrain = 16,
                       kStageFull = 17, kStageFree = 18, kNumBars = 19;
  static constexpr int kOffSlot = kOffBar + 8 * kNumBars;
  static constexpr int kOffAbort = kOffSlot + 4;
  static_assert(kOffAbort + 4 <= kOffBar + kBarArea, "barrier area too small");
  static constexpr uint32_t kTmemCols = 512;
  static __device__ __forceinline__ uint32_t col_s(int q) { return static_cast<uint32_t>(q & 1) * 128u; }
  static __device__ __forceinline__ uint32_t col_pv(int q) {
    return 256u + static_cast<uint32_t>(q & 1) * static_cast<uint32_t>(D);
  }
};

// First query tile that sees key tile j (all of them without the causal mask).
__device__ __forceinline__ int kv_outer_first_i(bool causal, int j) { return causal ? j : 0; }

template <int D, bool kCausal>
__global__ void __launch_bounds__(256, 1)
    kv_outer_fwd_kernel(const __grid_constant__ CUtensorMap tm_q,
                        const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_v,
                        const __grid_constant__ CUtensorMap tm_o, float* __restrict__ lse_out,
                        float* __restrict__ o_acc, float* __restrict__ m_ws,
                        float* __restrict__ l_ws, int n, int np, float scale_log2,
                        uint64_t limit_ns) {
  using L = KvOuterLayout<D>;
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
  const int bh = blockIdx.x;
  const int nt = np / 128;
  const unsigned int err_k = kErrFwd;

  if (threadIdx.x == 0) {
    for (int b = 0; b < L::kNumBars; ++b) {
      const bool four = (b >= L::kPReady && b < L::kPReady + 2) ||
                        (b >= L::kPvFree && b < L::kPvFree + 2) || b == L::kStageFull;
      mbar_init(bar(b), four ? 4u : 1u);
    }
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
      const uint32_t err = err_k | kErrRoleLoad;
      int q = 0, nkv = 0, nq = 0;
      bool ok = true;
      for (int j = 0; ok && j < nt; ++j) {
        const int kv = j & 1;
        if (!dbg_check(j * 128 < n, err, abort_flag) ||
            !wait_bounded(bar(L::kKvEmpty + kv), ((j >> 1) & 1) ^ 1, limit_ns, abort_flag, err))
          break;
        mbar_arrive_expect_tx(bar(L::kKvFull + kv), 2 * L::kTile);
        for (int db = 0; db < kDBlk; ++db) {
          tma_load_3d(sb + L::kOffK + kv * L::kTile + db * 16384, &tm_k, bar(L::kKvFull + kv),
                      db * 64, j * 128, bh);
          tma_load_3d(sb + L::kOffV + kv * L::kTile + db * 16384, &tm_v, bar(L::kKvFull + kv),
                      db * 64, j * 128, bh);
        }
        ++nkv;
        for (int i = kv_outer_first_i(kCausal, j); i < nt; ++i, ++q) {
          const int st = q & 1;
          if (!dbg_check(i * 128 < n, err, abort_flag) ||
              !wait_bounded(bar(L::kQEmpty + st), ((q >> 1) & 1) ^ 1, limit_ns, abort_flag, err)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(bar(L::kQFull + st), L::kTile);
          for (int db = 0; db < kDBlk; ++db)
            tma_load_3d(sb + L::kOffQ + st * L::kTile + db * 16384, &tm_q, bar(L::kQFull + st),
                        db * 64, i * 128, bh);
          ++nq;
        }
      }
      if (*abort_flag) {
        for (int x = (nkv > 2 ? nkv - 2 : 0); x < nkv; ++x)
          drain_wait(bar(L::kKvFull + (x & 1)), (x >> 1) & 1, limit_ns);
        for (int x = (nq > 2 ? nq - 2 : 0); x < nq; ++x)
          drain_wait(bar(L::kQFull + (x & 1)), (x >> 1) & 1, limit_ns);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // the whole warp runs this loop; the MMA and commit wrappers elect one lane
    {
      constexpr uint32_t id_s = idesc_bf16_f32(128, 128, false, false);
      constexpr uint32_t id_o = idesc_bf16_f32(128, D, false, true);
      const uint32_t err = err_k | kErrRoleMma;
      // P V of step q (key tile jq) once its P is ready; commits KvEmpty when
      // it is the last step of that key tile
      auto issue_pv = [&](int q, int jq, bool last_of_j) -> bool {
        if (!wait_bounded_warp(bar(L::kPReady + (q & 1)), (q >> 1) & 1, limit_ns, abort_flag, err) ||
            !wait_bounded_warp(bar(L::kPvFree + (q & 1)), ((q >> 1) & 1) ^ 1, limit_ns, abort_flag,
                               err))
          return false;
        tc_fence_after();
        const uint32_t va = sb + L::kOffV + (jq & 1) * L::kTile;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_bf16_ts(tmem + L::col_pv(q), tmem + L::col_s(q) + kk * 8,
                      sw128_desc(va + kk * 2048, 16384, 1024), id_o, kk > 0 ? 1u : 0u);
        tc_commit(bar(L::kPvFull + (q & 1)));
        if (last_of_j) tc_commit(bar(L::kKvEmpty + (jq & 1)));
        return true;
      };
      int q = 0;
      int prev_j = -1;
      bool prev_last = false, ok = true;
      for (int j = 0; ok && j < nt; ++j) {
        const int kv = j & 1;
        if (!wait_bounded_warp(bar(L::kKvFull + kv), (j >> 1) & 1, limit_ns, abort_flag, err)) break;
        const uint32_t ka = sb + L::kOffK + kv * L::kTile;
        const int i0 = kv_outer_first_i(kCausal, j);
        for (int i = i0; i < nt; ++i, ++q) {
          const int st = q & 1;
          if (!wait_bounded_warp(bar(L::kQFull + st), (q >> 1) & 1, limit_ns, abort_flag, err)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t qa = sb + L::kOffQ + st * L::kTile;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {  // S(q) = Q_i K_j^T (region q & 1 was last
            const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;  // read by P V(q - 2))
            mma_bf16_ss(tmem + L::col_s(q), sw128_desc(qa + off, 16, 1024),
                        sw128_desc(ka + off, 16, 1024), id_s, kk > 0 ? 1u : 0u);
          }
          tc_commit(bar(L::kSFull + st));
          tc_commit(bar(L::kQEmpty + st));
          if (q > 0 && !issue_pv(q - 1, prev_j, prev_last)) {
            ok = false;
            break;
          }
          prev_j = j;
          prev_last = (i == nt - 1);
        }
      }
      if (ok && q > 0) issue_pv(q - 1, prev_j, prev_last);
      tc_commit(bar(L::kDrain));
      drain_wait(bar(L::kDrain), 0, limit_ns);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ------------------------------------- softmax and O update (thread = row)
    const int r = threadIdx.x - 128;
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t err = err_k | kErrRoleSoftmax;
    int n_stores = 0;  // O tiles stored so far (phase of the staging barriers)
    // state of the step whose O update is pending
    float p_alpha = 0.f, p_beta = 0.f, p_m = 0.f, p_l = 0.f;
    int p_i = -1, p_j = -1, p_q = -1;
    bool ok = true;

    // O update of step pq (query tile pi, key tile pj): O = alpha O_old + beta P V.
    // After the last key tile of pi the result goes out as bf16 through the
    // staging tile: the four warps fill it (StageFull), warp 4 stores it with
    // TMA and frees it (StageFree) once the store has read it.  All waits are
    // bounded mbarrier waits, so a warp that gives up cannot hold the others.
    auto update_o = [&](int pq, int pi, int pj, float alpha, float beta, float m2, float l2) -> bool {
      const bool first = (pj == 0);
      const bool last = kCausal ? (pj == pi) : (pj == nt - 1);
      if (!wait_bounded_warp(bar(L::kPvFull + (pq & 1)), (pq >> 1) & 1, limit_ns, abort_flag, err))
        return false;
      if (last && !wait_bounded_warp(bar(L::kStageFree), (n_stores & 1) ^ 1, limit_ns, abort_flag,
                                     err))
        return false;
      tc_fence_after();
      const int row = pi * 128 + r;
      float* acc = o_acc + (static_cast<size_t>(bh) * nt + pi) * 128 * D + static_cast<size_t>(r) * 4;
      const uint32_t pv = tmem + lane_off + L::col_pv(pq);
      const uint32_t orow = sb + L::kOffStage + r * 128;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t u[32];
        tmem_ld_32x32b_x32(pv + c * 32, u);
        tmem_wait_ld_regs(u);
        float o[32];
#pragma unroll
        for (int g = 0; g < 8; ++g) {
          float4 old = make_float4(0.f, 0.f, 0.f, 0.f);
          if (!first) old = *reinterpret_cast<const float4*>(acc + (c * 8 + g) * 512);
          o[4 * g + 0] = fmaf(alpha, old.x, beta * __uint_as_float(u[4 * g + 0]));
          o[4 * g + 1] = fmaf(alpha, old.y, beta * __uint_as_float(u[4 * g + 1]));
          o[4 * g + 2] = fmaf(alpha, old.z, beta * __uint_as_float(u[4 * g + 2]));
          o[4 * g + 3] = fmaf(alpha, old.w, beta * __uint_as_float(u[4 * g + 3]));
        }
        if (last) {
#pragma unroll
          for (int qq = 0; qq < 4; ++qq) {
            const int jj = c * 4 + qq;  // 16-byte chunk of the output row
            st_shared_v4(orow + (jj >> 3) * 16384 + (((jj & 7) ^ (r & 7)) << 4),
                         pack_bf16x2(o[8 * qq + 0], o[8 * qq + 1]),
                         pack_bf16x2(o[8 * qq + 2], o[8 * qq + 3]),
                         pack_bf16x2(o[8 * qq + 4], o[8 * qq + 5]),
                         pack_bf16x2(o[8 * qq + 6], o[8 * qq + 7]));
          }
        } else {
#pragma unroll
          for (int g = 0; g < 8; ++g)
            *reinterpret_cast<float4*>(acc + (c * 8 + g) * 512) =
                make_float4(o[4 * g], o[4 * g + 1], o[4 * g + 2], o[4 * g + 3]);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(L::kPvFree + (pq & 1)));
      if (last) {
        if (row < n)
          lse_out[static_cast<size_t>(bh) * n + row] = (m2 + __log2f(l2)) * 0.69314718055994530942f;
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(L::kStageFull));
        if (warp == 4) {
          if (!wait_bounded_warp(bar(L::kStageFull), n_stores & 1, limit_ns, abort_flag, err))
            return false;
          if (lane == 0) {
            for (int db = 0; db < kDBlk; ++db)
              tma_store_3d(&tm_o, sb + L::kOffStage + db * 16384, db * 64, pi * 128, bh);
            bulk_commit_group();
            bulk_wait_group_read_0();  // the store has read the staging tile
            mbar_arrive(bar(L::kStageFree));
          }
          __syncwarp();
        }
        ++n_stores;
      }
      return true;
    };

    int q = 0;
    for (int j = 0; ok && j < nt; ++j) {
      for (int i = kv_outer_first_i(kCausal, j); i < nt; ++i, ++q) {
        if (!wait_bounded_warp(bar(L::kSFull + (q & 1)), (q >> 1) & 1, limit_ns, abort_flag, err)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t s_addr = tmem + lane_off + L::col_s(q);
        uint32_t u[128];
#pragma unroll
        for (int c = 0; c < 4; ++c)
          tmem_ld_32x32b_x32(s_addr + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&u[c * 32]));
        tmem_wait_ld_regs(u);
        int lim = 128;  // keys of this tile the row sees
        if (kCausal && j == i) lim = r + 1;
        const int rem = n - j * 128;
        if (rem < lim) lim = rem;
        // row max of c * s over the visible keys
        float mx = -INFINITY;
#pragma unroll
        for (int c = 0; c < 128; ++c) {
          const float x = __uint_as_float(u[c]) * scale_log2;
          mx = (c < lim) ? fmaxf(mx, x) : mx;
        }
        const size_t vrow = static_cast<size_t>(bh) * np + static_cast<size_t>(i) * 128 + r;
        const float m_old = (j == 0) ? -INFINITY : m_ws[vrow];
        const float l_old = (j == 0) ? 0.f : l_ws[vrow];
        const float m_new = fmaxf(m_old, mx);  // finite: every row sees key 0 at j = 0
        const float corr = (j == 0) ? 0.f : ex2_approx(m_old - m_new);
        float sum0 = 0.f, sum1 = 0.f;
#pragma unroll
        for (int qd = 0; qd < 4; ++qd) {
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            const int c = qd * 32 + e;
            float p0 = ex2_approx(fmaf(__uint_as_float(u[c]), scale_log2, -m_new));
            float p1 = ex2_approx(fmaf(__uint_as_float(u[c + 1]), scale_log2, -m_new));
            p0 = (c < lim) ? p0 : 0.f;
            p1 = (c + 1 < lim) ? p1 : 0.f;
            sum0 += p0;
            sum1 += p1;
            pk[e >> 1] = pack_bf16x2(p0, p1);
          }
          tmem_st_32x32b_x16(s_addr + qd * 16, pk);
        }
        const float l_new = fmaf(corr, l_old, sum0 + sum1);
        m_ws[vrow] = m_new;
        l_ws[vrow] = l_new;
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(L::kPReady + (q & 1)));
        // O update of the previous step while the tensor core runs this one's P V
        if (p_q >= 0 && !update_o(p_q, p_i, p_j, p_alpha, p_beta, p_m, p_l)) {
          ok = false;
          break;
        }
        const float inv_l = 1.0f / l_new;
        p_alpha = corr * l_old * inv_l;
        p_beta = inv_l;
        p_m = m_new;
        p_l = l_new;
        p_i = i;
        p_j = j;
        p_q = q;
      }
    }
    if (ok && p_q >= 0) update_o(p_q, p_i, p_j, p_alpha, p_beta, p_m, p_l);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, L::kTmemCols);
  }
}

}  // namespace fa
