// bwd.cuh -- backward attention kernels for sm_100a.
//
// The backward recomputes score tiles from Q, K and the saved row logsumexp
// instead of storing the N x N probability matrix (page "从零实现
// FlashAttention-2：分块在线 Softmax", section 反向传播：重算，而不是存储; page
// "FlashAttention为什么更快更省显存", section 反向传播为什么还要重算).  With
// P = exp(scale*S - LSE), dP = dO V^T, D_i = sum_c dO_ic O_ic and
// dS = P o (dP - D):  dV = P^T dO,  dK = scale dS^T Q,  dQ = scale dS K.
//
// Three launches:
//   bwd_preprocess_kernel : D = rowsum(dO o O), LSE in log2 units, clears the
//                           fp32 dQ accumulator (D / 8 lanes per row, reduced
//                           with warp shuffles)
//   bwd_main_kernel       : one CTA per 128-key tile owns dK_j and dV_j in TMEM
//                           (no atomics) and loops over the Q tiles that see
//                           it; dQ_i partial sums go to the fp32 accumulator
//                           with vector atomic adds
//   dq_convert_kernel     : dQ = bf16(scale * accumulator)
// The deterministic backward runs bwd_main_kernel without its dQ part, then
// dq_pass_kernel (dq_pass.cuh) in place of dq_convert_kernel: one CTA per
// 128-row Q tile sums dQ over the key tiles in a fixed order and writes it.
#pragma once

#include <cuda_bf16.h>

#include "common.cuh"

namespace fa {

// ------------------------------------------------------------ preprocess
// rows = BH * np (< 2^31: the tensors fit in device memory); row r of slice
// bh is valid iff r < n.  D / 8 lanes share a row (one 16-byte load of O and
// of dO each, reduced with warp shuffles); a warp takes 32 / (D / 8) rows per
// step and kUnroll steps at once, issuing all of their loads before the first
// reduction, and strides over the rows with the whole grid.
template <int D>
__global__ void __launch_bounds__(256)
    bwd_preprocess_kernel(const __nv_bfloat16* __restrict__ o, const __nv_bfloat16* __restrict__ dout,
                          const float* __restrict__ lse, float* __restrict__ dvec,
                          float* __restrict__ lse2, float* __restrict__ dq_acc, int bh_count, int n,
                          int np, float log2e) {
  constexpr int kLanes = D / 8;               // lanes per row
  constexpr int kRowsPerStep = 32 / kLanes;   // rows per warp and step
  constexpr int kUnroll = 4;
  constexpr int kRowsPerWarp = kRowsPerStep * kUnroll;
  const uint32_t total = static_cast<uint32_t>(bh_count) * static_cast<uint32_t>(np);
  const uint32_t unp = static_cast<uint32_t>(np), un = static_cast<uint32_t>(n);
  const int lane = threadIdx.x & 31;
  const uint32_t sub = static_cast<uint32_t>(lane / kLanes);  // row within the step
  const int cl = lane % kLanes;                                // 8-element chunk of the row
  const uint32_t warps = (gridDim.x * blockDim.x) >> 5;
  for (uint32_t w = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; w * kRowsPerWarp < total;
       w += warps) {  // warp-uniform loop
    const uint32_t row0 = w * kRowsPerWarp;
    uint4 a[kUnroll], b[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const uint32_t vr = row0 + u * kRowsPerStep + sub;
      const uint32_t bh = vr / unp, r = vr - bh * unp;
      a[u] = make_uint4(0u, 0u, 0u, 0u);
      b[u] = a[u];
      if (vr < total && r < un) {
        const size_t base = (static_cast<size_t>(bh) * un + r) * D + cl * 8;
        a[u] = *reinterpret_cast<const uint4*>(o + base);
        b[u] = *reinterpret_cast<const uint4*>(dout + base);
      }
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const uint32_t av[4] = {a[u].x, a[u].y, a[u].z, a[u].w};
      const uint32_t bv[4] = {b[u].x, b[u].y, b[u].z, b[u].w};
      float acc = 0.f;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        acc = fmaf(bf16_lo(av[i]), bf16_lo(bv[i]), acc);
        acc = fmaf(bf16_hi(av[i]), bf16_hi(bv[i]), acc);
      }
#pragma unroll
      for (int off = kLanes / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
      const uint32_t vr = row0 + u * kRowsPerStep + sub;
      if (vr < total) {
        const uint32_t bh = vr / unp, r = vr - bh * unp;
        if (cl == 0) {
          dvec[vr] = acc;
          // rows past the end get +inf so that their recomputed probabilities are 0
          lse2[vr] = (r < un) ? lse[static_cast<size_t>(bh) * un + r] * log2e : INFINITY;
        }
        if (dq_acc != nullptr) {  // the deterministic backward has no accumulator
          float4* acc_row = reinterpret_cast<float4*>(dq_acc + static_cast<size_t>(vr) * D) + cl * 2;
          acc_row[0] = make_float4(0.f, 0.f, 0.f, 0.f);
          acc_row[1] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
      }
    }
  }
}

// ------------------------------------------------------------- dQ convert
// The accumulator holds each 128-row tile as [D/4 column groups][128 rows][4].
// A warp covers 16 consecutive rows and two adjacent 8-column chunks p, p + 1:
// lane pair (2k, 2k + 1) writes the 32 contiguous bytes of row k (one full
// sector), and for each of the four column groups read, the warp's 16 rows are
// 256 contiguous bytes.
template <int D>
__global__ void __launch_bounds__(256)
    dq_convert_kernel(const float* __restrict__ dq_acc, __nv_bfloat16* __restrict__ dq, int bh_count,
                      int n, int np, float scale) {
  constexpr int kPairs = D / 16;  // chunk pairs per row
  const long long gw = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const long long row_blocks = (static_cast<long long>(bh_count) * n + 15) / 16;
  if (gw >= row_blocks * kPairs) return;
  const int cp = static_cast<int>(gw % kPairs);
  const long long row = (gw / kPairs) * 16 + (lane >> 1);  // bh * n + r
  if (row >= static_cast<long long>(bh_count) * n) return;
  const int p = 2 * cp + (lane & 1);  // 8-column chunk
  const long long bh = row / n;
  const int r = static_cast<int>(row % n);
  const float* tile = dq_acc + (bh * (np / 128) + r / 128) * 128LL * D;
  const float4 x = *reinterpret_cast<const float4*>(tile + (2 * p) * 512 + (r % 128) * 4);
  const float4 y = *reinterpret_cast<const float4*>(tile + (2 * p + 1) * 512 + (r % 128) * 4);
  uint4 w;
  w.x = pack_bf16x2(x.x * scale, x.y * scale);
  w.y = pack_bf16x2(x.z * scale, x.w * scale);
  w.z = pack_bf16x2(y.x * scale, y.y * scale);
  w.w = pack_bf16x2(y.z * scale, y.w * scale);
  *reinterpret_cast<uint4*>(dq + row * D + 8 * p) = w;
}

}  // namespace fa

#include "bwd_main.cuh"
#include "dq_pass.cuh"
