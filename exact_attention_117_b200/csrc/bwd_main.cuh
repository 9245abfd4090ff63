#pragma once
namespace fa {
template <int D>
struct BwdLayout {
  static constexpr int kThreads = 256;
  static constexpr int kSmemAlloc = 1024;
};
template <int D, bool kCausal>
__global__ void bwd_main_kernel(const __grid_constant__ CUtensorMap, const __grid_constant__ CUtensorMap,
                                const __grid_constant__ CUtensorMap, const __grid_constant__ CUtensorMap,
                                const float*, const float*, float*, __nv_bfloat16*, __nv_bfloat16*,
                                int, int, float, float, uint64_t) {}
}  // namespace fa
