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
//                           fp32 dQ accumulator (one warp per row, reduced
//                           with warp shuffles)
//   bwd_main_kernel       : one CTA per 128-key tile owns dK_j and dV_j in TMEM
//                           (no atomics) and loops over the Q tiles that see
//                           it; dQ_i partial sums go to the fp32 accumulator
//                           with vector atomic adds
//   dq_convert_kernel     : dQ = bf16(scale * accumulator)
#pragma once

#include <cuda_bf16.h>

#include "common.cuh"

namespace fa {

// ------------------------------------------------------------ preprocess
// rows = BH * np; row r of slice bh is valid iff r < n.  One warp per row.
template <int D>
__global__ void __launch_bounds__(256)
    bwd_preprocess_kernel(const __nv_bfloat16* __restrict__ o, const __nv_bfloat16* __restrict__ dout,
                          const float* __restrict__ lse, float* __restrict__ dvec,
                          float* __restrict__ lse2, float* __restrict__ dq_acc, int bh_count, int n,
                          int np, float log2e) {
  const long long gw = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (gw >= static_cast<long long>(bh_count) * np) return;
  const int bh = static_cast<int>(gw / np);
  const int r = static_cast<int>(gw % np);
  constexpr int kPer = D / 32;  // elements per lane: 2 or 4
  float acc = 0.f;
  if (r < n) {
    const size_t base = (static_cast<size_t>(bh) * n + r) * D + lane * kPer;
    if constexpr (kPer == 4) {
      const uint2 a = *reinterpret_cast<const uint2*>(o + base);
      const uint2 b = *reinterpret_cast<const uint2*>(dout + base);
      const __nv_bfloat162* a2 = reinterpret_cast<const __nv_bfloat162*>(&a);
      const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&b);
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const float2 fa2 = __bfloat1622float2(a2[i]);
        const float2 fb2 = __bfloat1622float2(b2[i]);
        acc = fmaf(fa2.x, fb2.x, acc);
        acc = fmaf(fa2.y, fb2.y, acc);
      }
    } else {
      const __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162*>(o + base);
      const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162*>(dout + base);
      const float2 fa2 = __bfloat1622float2(a);
      const float2 fb2 = __bfloat1622float2(b);
      acc = fmaf(fa2.x, fb2.x, acc);
      acc = fmaf(fa2.y, fb2.y, acc);
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  const size_t vrow = static_cast<size_t>(bh) * np + r;
  if (lane == 0) {
    dvec[vrow] = acc;
    // rows past the end get +inf so that their recomputed probabilities are 0
    lse2[vrow] = (r < n) ? lse[static_cast<size_t>(bh) * n + r] * log2e : INFINITY;
  }
  if (dq_acc != nullptr) {  // the deterministic backward has no accumulator
    float4* acc_row = reinterpret_cast<float4*>(dq_acc + vrow * D);
    const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int i = lane; i < D / 4; i += 32) acc_row[i] = z;
  }
}

// ------------------------------------------------------------- dQ convert
// The accumulator holds each 128-row tile as [D/4 column groups][128 rows][4];
// thread (p, row) reads column groups 2p and 2p+1 of its row (consecutive
// threads take consecutive rows: coalesced reads) and writes 8 bf16 of dQ.
template <int D>
__global__ void __launch_bounds__(256)
    dq_convert_kernel(const float* __restrict__ dq_acc, __nv_bfloat16* __restrict__ dq, int bh_count,
                      int n, int np, float scale) {
  const long long idx = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const long long rows = static_cast<long long>(bh_count) * n;
  if (idx >= rows * (D / 8)) return;
  const int p = static_cast<int>(idx / rows);  // group of 8 columns
  const long long row = idx % rows;            // bh * n + r
  const long long bh = row / n;
  const int r = static_cast<int>(row % n);
  const float* tile = dq_acc + (bh * (np / 128) + r / 128) * 128LL * D;
  const float4 a = *reinterpret_cast<const float4*>(tile + (2 * p) * 512 + (r % 128) * 4);
  const float4 b = *reinterpret_cast<const float4*>(tile + (2 * p + 1) * 512 + (r % 128) * 4);
  uint4 w;
  w.x = pack_bf16x2(a.x * scale, a.y * scale);
  w.y = pack_bf16x2(a.z * scale, a.w * scale);
  w.z = pack_bf16x2(b.x * scale, b.y * scale);
  w.w = pack_bf16x2(b.z * scale, b.w * scale);
  *reinterpret_cast<uint4*>(dq + row * D + 8 * p) = w;
}

}  // namespace fa

#include "bwd_main.cuh"
#include "dq_pass.cuh"
