// fwd.cuh -- forward attention kernel for sm_100a.
//
// Algorithm (page "从零实现 FlashAttention-2：分块在线 Softmax", sections
// 在线 softmax：重缩放恒等式 and 从 FlashAttention-1 到 FlashAttention-2; page
// "FlashAttention 为什么能节省显存并提速,是否改变注意力结果?", section
// 难点在于分块后softmax如何归一): one CTA owns one 128-row Q tile of one
// (batch, head).  The Q tile stays in shared memory; 128-key K/V tiles stream
// through a TMA ring; per key tile the CTA computes S = Q K^T on the tensor
// cores into TMEM, updates the running row max m and sum l, rescales the
// output accumulator by exp(m_old - m_new) when the max moved (the factor is
// exactly 1 otherwise: page 2, section 提示), and accumulates O += P V on the
// tensor cores.  O / l and the row logsumexp are written once at the end; no
// N x N tensor ever reaches global memory.
//
// Causal masking (page 2, section 提示): key tiles wholly above the diagonal
// are never loaded; the diagonal tile masks key > query inside the tile.
//
// Warp roles (256 threads):
//   warp 0     : TMA producer (Q once, then K_j / V_j into a kStages ring)
//   warp 1     : TMEM allocator and tcgen05.mma issuer
//   warps 2-3  : idle
//   warps 4-7  : softmax / rescale / epilogue, one thread per query row
//                (TMEM lane = row, so the row max and row sum stay inside one
//                thread and need no cross-lane reduction)
//
// TMEM columns: S double buffer at [0,128) and [128,256), O at [256, 256+D).
// All exponentials are base 2 with scale*log2(e) folded in; the stored LSE is
// converted back to natural log.
#pragma once

#include "common.cuh"

namespace fa {

template <int D>
struct FwdLayout {
  static constexpr int kBM = 128;                    // query rows per tile
  static constexpr int kBN = 128;                    // keys per tile
  static constexpr int kStages = (D == 64) ? 3 : 2;  // K/V ring depth
  static constexpr int kTile = kBM * D * 2;          // bytes of a Q, K or V tile
  static constexpr int kPTile = kBM * kBN * 2;       // bytes of the bf16 P tile
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kOffQ + kTile;
  static constexpr int kOffV = kOffK + kStages * kTile;
  static constexpr int kOffP = kOffV + kStages * kTile;
  static constexpr int kOffBar = kOffP + kPTile;
  static constexpr int kBarArea = 256;
  static constexpr int kBytes = kOffBar + kBarArea;
  static constexpr int kSmemAlloc = kBytes + 1024;  // slack to align the base to 1 KiB
  // barrier indices
  static constexpr int kQFull = 0;
  static constexpr int kKFull = 1;
  static constexpr int kKEmpty = kKFull + kStages;
  static constexpr int kVFull = kKEmpty + kStages;
  static constexpr int kVEmpty = kVFull + kStages;
  static constexpr int kSFull = kVEmpty + kStages;  // 2
  static constexpr int kSFree = kSFull + 2;         // 2
  static constexpr int kPFull = kSFree + 2;
  static constexpr int kODone = kPFull + 1;
  static constexpr int kDrain = kODone + 1;
  static constexpr int kNumBars = kDrain + 1;
  static constexpr int kOffSlot = kOffBar + 8 * kNumBars;  // TMEM base address
  static constexpr int kOffAbort = kOffSlot + 4;
  static_assert(kOffAbort + 4 <= kOffBar + kBarArea, "barrier area too small");
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kColS0 = 0, kColS1 = 128, kColO = 256;
};

template <int D, bool kCausal>
__global__ void __launch_bounds__(256, 1)
    fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
               const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
               float* __restrict__ lse_out, int n, float scale_log2, uint64_t limit_ns) {
  using L = FwdLayout<D>;
  constexpr int S = L::kStages;
  constexpr int kDBlk = D / 64;  // 128-byte swizzle blocks per tile row

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
  const int qt = static_cast<int>(gridDim.y) - 1 - static_cast<int>(blockIdx.y);  // heavy first
  const int n_kv = kCausal ? (qt + 1) : (n + L::kBN - 1) / L::kBN;
  const unsigned int err_fwd = kErrFwd;

  if (threadIdx.x == 0) {
    mbar_init(bar(L::kQFull), 1);
    for (int s = 0; s < S; ++s) {
      mbar_init(bar(L::kKFull + s), 1);
      mbar_init(bar(L::kKEmpty + s), 1);
      mbar_init(bar(L::kVFull + s), 1);
      mbar_init(bar(L::kVEmpty + s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar(L::kSFull + b), 1);
      mbar_init(bar(L::kSFree + b), 4);  // one arrive per softmax warp
    }
    mbar_init(bar(L::kPFull), 4);
    mbar_init(bar(L::kODone), 1);
    mbar_init(bar(L::kDrain), 1);
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
      tma_prefetch_desc(&tm_o);
      bool ok = true;
      int issued = 0;
      mbar_arrive_expect_tx(bar(L::kQFull), L::kTile);
      for (int db = 0; db < kDBlk; ++db)
        tma_load_3d(sb + L::kOffQ + db * 16384, &tm_q, bar(L::kQFull), db * 64, qt * L::kBM, bh);
      for (int t = 0; t < n_kv; ++t) {
        const int s = t % S;
        const uint32_t ph = (t / S) & 1;
        if (!wait_bounded(bar(L::kKEmpty + s), ph ^ 1, limit_ns, abort_flag,
                          err_fwd | kErrRoleLoad)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(bar(L::kKFull + s), L::kTile);
        for (int db = 0; db < kDBlk; ++db)
          tma_load_3d(sb + L::kOffK + s * L::kTile + db * 16384, &tm_k, bar(L::kKFull + s),
                      db * 64, t * L::kBN, bh);
        if (!wait_bounded(bar(L::kVEmpty + s), ph ^ 1, limit_ns, abort_flag,
                          err_fwd | kErrRoleLoad)) {
          ok = false;
          issued = 2 * t + 1;
          break;
        }
        mbar_arrive_expect_tx(bar(L::kVFull + s), L::kTile);
        for (int db = 0; db < kDBlk; ++db)
          tma_load_3d(sb + L::kOffV + s * L::kTile + db * 16384, &tm_v, bar(L::kVFull + s),
                      db * 64, t * L::kBN, bh);
        issued = 2 * t + 2;
      }
      if (!ok) {
        // let every copy already issued land before shared memory is released
        drain_wait(bar(L::kQFull), 0, limit_ns);
        const int nk = (issued + 1) / 2, nv = issued / 2;
        for (int t = (nk > S ? nk - S : 0); t < nk; ++t)
          drain_wait(bar(L::kKFull + t % S), (t / S) & 1, limit_ns);
        for (int t = (nv > S ? nv - S : 0); t < nv; ++t)
          drain_wait(bar(L::kVFull + t % S), (t / S) & 1, limit_ns);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t id_s = idesc_bf16_f32(128, 128, false, false);
      constexpr uint32_t id_o = idesc_bf16_f32(128, D, false, true);
      const uint32_t err = err_fwd | kErrRoleMma;
      auto issue_s = [&](int t) -> bool {
        const int s = t % S;
        const int b = t & 1;
        if (!wait_bounded(bar(L::kKFull + s), (t / S) & 1, limit_ns, abort_flag, err)) return false;
        if (!wait_bounded(bar(L::kSFree + b), ((t >> 1) & 1) ^ 1, limit_ns, abort_flag, err))
          return false;
        tc_fence_after();
        const uint32_t qa = sb + L::kOffQ;
        const uint32_t ka = sb + L::kOffK + s * L::kTile;
        const uint32_t d_tmem = tmem + (b ? L::kColS1 : L::kColS0);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
          mma_bf16_ss(d_tmem, sw128_desc(qa + off, 16, 1024), sw128_desc(ka + off, 16, 1024), id_s,
                      kk > 0 ? 1u : 0u);
        }
        tc_commit(bar(L::kSFull + b));
        tc_commit(bar(L::kKEmpty + s));
        return true;
      };
      bool ok = wait_bounded(bar(L::kQFull), 0, limit_ns, abort_flag, err) && issue_s(0);
      for (int t = 0; ok && t < n_kv; ++t) {
        if (t + 1 < n_kv && !issue_s(t + 1)) break;
        const int s = t % S;
        if (!wait_bounded(bar(L::kPFull), t & 1, limit_ns, abort_flag, err)) break;
        if (!wait_bounded(bar(L::kVFull + s), (t / S) & 1, limit_ns, abort_flag, err)) break;
        tc_fence_after();
        const uint32_t pa = sb + L::kOffP;
        const uint32_t va = sb + L::kOffV + s * L::kTile;
#pragma unroll
        for (int kk = 0; kk < L::kBN / 16; ++kk) {
          const uint32_t poff = (kk >> 2) * 16384 + (kk & 3) * 32;
          mma_bf16_ss(tmem + L::kColO, sw128_desc(pa + poff, 16, 1024),
                      sw128_desc(va + kk * 2048, 16384, 1024), id_o, (t > 0 || kk > 0) ? 1u : 0u);
        }
        tc_commit(bar(L::kODone));
        tc_commit(bar(L::kVEmpty + s));
      }
      // every MMA issued above must finish before TMEM / smem are released
      tc_commit(bar(L::kDrain));
      drain_wait(bar(L::kDrain), 0, limit_ns);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ------------------------------------------------- softmax / epilogue
    const int r = threadIdx.x - 128;  // row inside the tile == TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t err = err_fwd | kErrRoleSoftmax;
    float m_run = -INFINITY;  // running max of scale*log2(e)*s
    float l_run = 0.f;        // running sum of 2^(x - m_run)
    bool ok = true;
    for (int t = 0; t < n_kv; ++t) {
      const int b = t & 1;
      if (!wait_bounded(bar(L::kSFull + b), (t >> 1) & 1, limit_ns, abort_flag, err)) {
        ok = false;
        break;
      }
      tc_fence_after();
      float x[128];
      {
        const uint32_t sa = tmem + lane_off + (b ? L::kColS1 : L::kColS0);
        uint32_t u[128];
#pragma unroll
        for (int c = 0; c < 4; ++c)
          tmem_ld_32x32b_x32(sa + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&u[c * 32]));
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 128; ++i) x[i] = __uint_as_float(u[i]) * scale_log2;
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(L::kSFree + b));

      // mask: causal diagonal tile (key > query) and keys past the end
      int lim = L::kBN;
      if (kCausal && t == qt) lim = r + 1;
      const int rem = n - t * L::kBN;
      if (rem < lim) lim = rem;
      if (lim < L::kBN) {
#pragma unroll
        for (int c = 0; c < 128; ++c) x[c] = (c < lim) ? x[c] : -INFINITY;
      }
      float mx0 = x[0], mx1 = x[1], mx2 = x[2], mx3 = x[3];
#pragma unroll
      for (int c = 4; c < 128; c += 4) {
        mx0 = fmaxf(mx0, x[c]);
        mx1 = fmaxf(mx1, x[c + 1]);
        mx2 = fmaxf(mx2, x[c + 2]);
        mx3 = fmaxf(mx3, x[c + 3]);
      }
      const float m_new = fmaxf(m_run, fmaxf(fmaxf(mx0, mx1), fmaxf(mx2, mx3)));
      const float alpha = ex2_approx(m_run - m_new);
      uint32_t pk[64];
      float sum0 = 0.f, sum1 = 0.f;
#pragma unroll
      for (int c = 0; c < 128; c += 2) {
        const float p0 = ex2_approx(x[c] - m_new);
        const float p1 = ex2_approx(x[c + 1] - m_new);
        sum0 += p0;
        sum1 += p1;
        pk[c >> 1] = pack_bf16x2(p0, p1);
      }
      l_run = l_run * alpha + (sum0 + sum1);
      m_run = m_new;

      if (t > 0) {
        // PV of the previous tile must be done: it reads P and accumulates O
        if (!wait_bounded(bar(L::kODone), (t - 1) & 1, limit_ns, abort_flag, err)) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (__any_sync(0xffffffffu, alpha != 1.0f)) {
          const uint32_t oa = tmem + lane_off + L::kColO;
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t u[32];
            tmem_ld_32x32b_x32(oa + c * 32, u);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) u[i] = __float_as_uint(__uint_as_float(u[i]) * alpha);
            tmem_st_32x32b_x32(oa + c * 32, u);
          }
          tmem_wait_st();
        }
      }
      // P tile: K-major, 128-byte swizzle, two 64-key blocks of 16 KiB
      {
        const uint32_t prow = sb + L::kOffP + r * 128;
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const uint32_t addr = prow + (j >> 3) * 16384 + ((((j & 7) ^ (r & 7))) << 4);
          st_shared_v4(addr, pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(L::kPFull));
    }

    // ------------------------------------------------------------ epilogue
    if (ok) ok = wait_bounded(bar(L::kODone), (n_kv - 1) & 1, limit_ns, abort_flag,
                              err_fwd | kErrRoleEpilogue);
    if (ok) {
      tc_fence_after();
      const float inv_l = 1.0f / l_run;
      const uint32_t oa = tmem + lane_off + L::kColO;
      const uint32_t orow = sb + L::kOffQ + r * 128;  // Q tile is dead: stage O there
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t u[32];
        tmem_ld_32x32b_x32(oa + c * 32, u);
        tmem_wait_ld();
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int j = c * 4 + q;  // 16-byte chunk index within the row
          const uint32_t addr = orow + (j >> 3) * 16384 + ((((j & 7) ^ (r & 7))) << 4);
          st_shared_v4(addr,
                       pack_bf16x2(__uint_as_float(u[8 * q + 0]) * inv_l,
                                   __uint_as_float(u[8 * q + 1]) * inv_l),
                       pack_bf16x2(__uint_as_float(u[8 * q + 2]) * inv_l,
                                   __uint_as_float(u[8 * q + 3]) * inv_l),
                       pack_bf16x2(__uint_as_float(u[8 * q + 4]) * inv_l,
                                   __uint_as_float(u[8 * q + 5]) * inv_l),
                       pack_bf16x2(__uint_as_float(u[8 * q + 6]) * inv_l,
                                   __uint_as_float(u[8 * q + 7]) * inv_l));
        }
      }
      const int row = qt * L::kBM + r;
      if (row < n) lse_out[static_cast<size_t>(bh) * n + row] = (m_run + __log2f(l_run)) * 0.69314718055994530942f;
      fence_proxy_async_smem();
    }
    tc_fence_before();
    named_barrier_sync(1, 128);  // every softmax warp reaches this, ok or not
    if (threadIdx.x == 128 && ok && !*abort_flag) {
      for (int db = 0; db < kDBlk; ++db)
        tma_store_3d(&tm_o, sb + L::kOffQ + db * 16384, db * 64, qt * L::kBM, bh);
      bulk_commit_group();
      bulk_wait_group_0();
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
