// fa_api.cu -- the C ABI declared in include/fa.h: argument checks, TMA
// descriptor encoding, kernel selection and launch, error word, timing.
//
// This is the only translation unit of the library: the kernels are included
// from their headers so that they can all name the one device error word.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <vector>

#include "../../include/fa.h"
#include "bwd.cuh"
#include "fwd.cuh"
#include "kv_outer.cuh"

namespace {

constexpr int kMaxDevices = 64;
constexpr int kMaxSplits = 64;
constexpr uint64_t kWaitLimitNs = 4000000000ull;  // 4 s per bounded wait

// ------------------------------------------------------------ TMA encoding
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// bf16 tensor [BH, rows, cols] (cols innermost), box = box_cols cols x box_rows
// rows x 1.  Out-of-range loads read zeros; stores are clipped.
bool encode_bf16_3d_box(CUtensorMap* map, const void* ptr, int cols, int rows, int bh,
                        int box_cols, int box_rows, CUtensorMapSwizzle swizzle) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows),
                        static_cast<cuuint64_t>(bh)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(cols) * 2,
                           static_cast<cuuint64_t>(cols) * 2 * static_cast<cuuint64_t>(rows)};
  cuuint32_t box[3] = {static_cast<cuuint32_t>(box_cols), static_cast<cuuint32_t>(box_rows), 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// The operand layout of the kernels: 64 cols (128 bytes) x box_rows, 128-byte swizzle.
bool encode_bf16_3d(CUtensorMap* map, const void* ptr, int cols, int rows, int bh, int box_rows) {
  return encode_bf16_3d_box(map, ptr, cols, rows, bh, 64, box_rows, CU_TENSOR_MAP_SWIZZLE_128B);
}

// Outputs stored from per-warp staging boxes (the forward's O, the backward's
// dK and dV): 32 x 32 boxes (64-byte rows), 64-byte swizzle
// (fa::FwdLayout::kOffStage, fa::BwdLayout::kOffStage).
bool encode_out_box32(CUtensorMap* map, const void* o, int d, int N, int bh) {
  return encode_bf16_3d_box(map, o, d, N, bh, 32, 32, CU_TENSOR_MAP_SWIZZLE_64B);
}

// --------------------------------------------------------------- timing
struct TimedLaunch {
  int kernel;
  cudaEvent_t start, stop;
};
struct Timing {
  std::mutex mu;
  bool active = false;
  std::vector<TimedLaunch> launches;
  std::vector<cudaEvent_t> pool;
} g_timing;

constexpr size_t kMaxTimed = 65536;

cudaEvent_t pool_event() {
  if (!g_timing.pool.empty()) {
    cudaEvent_t e = g_timing.pool.back();
    g_timing.pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
  return e;
}

// Brackets one launch with events when a timing session is open.
struct LaunchTimer {
  cudaStream_t stream;
  int kernel;
  cudaEvent_t start = nullptr, stop = nullptr;
  LaunchTimer(cudaStream_t s, int k) : stream(s), kernel(k) {
    std::lock_guard<std::mutex> lock(g_timing.mu);
    if (!g_timing.active || g_timing.launches.size() >= kMaxTimed) return;
    start = pool_event();
    stop = pool_event();
    if (start && stop) cudaEventRecord(start, stream);
  }
  ~LaunchTimer() {
    if (!(start && stop)) return;
    cudaEventRecord(stop, stream);
    std::lock_guard<std::mutex> lock(g_timing.mu);
    g_timing.launches.push_back({kernel, start, stop});
  }
};

// ------------------------------------------------------------ helpers
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

fa_status check_common(int B, int H, int N, int d, float scale) {
  if (B < 1 || H < 1 || N < 1) return FA_ERR_SHAPE;
  const long long bh = static_cast<long long>(B) * H;
  if (bh > 0x7fffffffLL) return FA_ERR_SHAPE;
  // sequence length bound (8.4 M rows), far beyond what fits in device memory
  // at any B*H: row and tile indices stay well inside 32-bit arithmetic
  if (N > (65535 * 128)) return FA_ERR_SHAPE;
  // the backward main kernel numbers its B*H*ceil(N/128) work items, and the
  // kernels index blocks and items with 32-bit signed arithmetic
  if (bh * ((static_cast<long long>(N) + 127) / 128) > 0x7fffffffLL) return FA_ERR_SHAPE;
  if (static_cast<long long>(N) * bh > (1LL << 40)) return FA_ERR_SHAPE;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED_D;
  if (!std::isfinite(scale)) return FA_ERR_SCALE;
  return FA_OK;
}

template <typename K>
bool set_smem(K kernel, int bytes) {
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) ==
         cudaSuccess;
}

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Number of SMs of device `dev` (looked up once per device).
int sm_count(int dev) {
  static int count[kMaxDevices] = {};
  if (dev < 0 || dev >= kMaxDevices) return 148;
  if (count[dev] == 0) {
    int c = 0;
    if (cudaDeviceGetAttribute(&c, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || c <= 0)
      c = 148;
    count[dev] = c;
  }
  return count[dev];
}

struct BwdWorkspace {
  float* dq_acc;  // [BH, Np, d]
  float* dvec;    // [BH, Np]
  float* lse2;    // [BH, Np]
  size_t bytes;
};

BwdWorkspace bwd_workspace_layout(void* base, int B, int H, int N, int d) {
  const size_t bh = static_cast<size_t>(B) * H;
  const size_t np = round_up(static_cast<size_t>(N), 128);
  const size_t acc = bh * np * d * sizeof(float);
  const size_t vec = round_up(bh * np * sizeof(float), 256);
  char* p = static_cast<char*>(base);
  BwdWorkspace w;
  w.dq_acc = reinterpret_cast<float*>(p);
  w.dvec = reinterpret_cast<float*>(p + acc);
  w.lse2 = reinterpret_cast<float*>(p + acc + vec);
  w.bytes = acc + 2 * vec;
  return w;
}

// Per-device launch sequence numbers: a persistent kernel's launch takes work
// counter slot (sequence mod kSchedSlots) (see common.cuh).
std::atomic<uint32_t> g_launch_seq[kMaxDevices];

uint32_t next_sched_slot(int dev) {
  return g_launch_seq[dev].fetch_add(1u) & static_cast<uint32_t>(fa::kSchedSlots - 1);
}

template <int D, bool C, bool kSplit>
fa_status launch_fwd(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                     const CUtensorMap& mo, float* lse, int BH, int N, float scale_log2,
                     cudaStream_t st,
                     int num_splits = 1, float* part_o = nullptr, float* part_lse = nullptr) {
  using L = fa::FwdLayout<D>;
  static bool attr_set[kMaxDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return FA_ERR_CUDA;
  if (!attr_set[dev]) {
    if (!set_smem(fa::fwd_kernel<D, C, kSplit>, L::kSmemAlloc)) return FA_ERR_CUDA;
    attr_set[dev] = true;
  }
  const int q_tiles = (N + L::kBM - 1) / L::kBM;
  const int pairs = (q_tiles + 1) / 2;
  // Work items: (head, pair of Q tiles[, split]).  The heads go in
  // launch-order groups whose K and V (4 N d bytes per head) come to about
  // 32 MB, 8 to 128 heads (fewer if there are fewer), which the busy CTAs
  // share in L2 (B200, causal, against a fixed 32 heads: B*H*N = 2^20 at
  // N = 512 d = 128 128 heads 505 vs 468 TFLOP/s, N = 8192 8 heads 1172 vs
  // 1124; B=1 H=32 N=16384 8 heads 1234 vs 1176; B=2 H=16 N=4096 16 heads
  // as fast as 32; within 2 % of the best size at N = 1024 / 2048, d = 64).
  const long long kv_bytes = 4LL * q_tiles * L::kBM * D;
  const int head_group =
      static_cast<int>(std::max(8LL, std::min(128LL, (32LL << 20) / kv_bytes)));
  const long long items = static_cast<long long>(BH) * pairs * (kSplit ? num_splits : 1);
  if (items > 0x7fffffffLL) return FA_ERR_SHAPE;
  const int n_items = static_cast<int>(items);
  const int grid = std::min(n_items, sm_count(dev));  // persistent: one CTA per SM
  const uint32_t slot = next_sched_slot(dev);
  // the kernel's masked score (-inf after scaling) needs a nonzero factor; at
  // 1e-30 every scaled score of a finite input is 0 to fp32 accuracy, as it is
  // for a zero scale
  if (std::fabs(scale_log2) < 1e-30f) scale_log2 = std::signbit(scale_log2) ? -1e-30f : 1e-30f;
  {
    LaunchTimer timer(st, FA_KERNEL_FWD);
    fa::fwd_kernel<D, C, kSplit><<<grid, 384, L::kSmemAlloc, st>>>(
        mq, mk, mv, mo, lse, N, BH, scale_log2, kWaitLimitNs,
        num_splits, part_o, part_lse, head_group, n_items, slot);
  }
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

// Heads per launch-order group of the backward main kernel.  The busy CTAs
// share the Q, dO and fp32 dQ accumulator tiles of a group through L2, 8 N d
// bytes per head; groups of about kBwdGroupBytes, 4 to 64 heads, measured
// best among 32, 64 and 128 MB and a fixed 8 heads (B200, causal, atomic
// backward main kernel, 64 MB against 8 heads: B=128 H=16 N=512 560 vs 502
// TFLOP/s, B=16 H=16 N=4096 d=64 667 vs 591, B=1 H=32 N=16384 1023 vs 981,
// B=2 H=16 N=4096 981 vs 968; the deterministic one unchanged).
constexpr long long kBwdGroupBytes = 64LL << 20;
int bwd_head_group(int BH, int np, int d) {
  const long long per_head = 8LL * np * d;
  const long long g = std::max(4LL, std::min(64LL, kBwdGroupBytes / per_head));
  return static_cast<int>(std::min<long long>(g, BH));
}

template <int D, bool C, bool kDet>
fa_status launch_bwd(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                     const CUtensorMap& mdo, const CUtensorMap& mdk, const CUtensorMap& mdv,
                     const CUtensorMap& mdq, const void* o, const void* dout, const float* lse,
                     void* dq, const BwdWorkspace& ws, int BH, int N, float scale,
                     cudaStream_t st) {
  using L = fa::BwdLayout<D>;
  using LQ = fa::DqLayout<D>;
  static bool attr_set[kMaxDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev >= kMaxDevices) return FA_ERR_CUDA;
  if (!attr_set[dev]) {
    if (!set_smem(fa::bwd_main_kernel<D, C, !kDet>, L::kSmemAlloc)) return FA_ERR_CUDA;
    if (kDet && !set_smem(fa::dq_pass_kernel<D, C>, LQ::kSmemAlloc)) return FA_ERR_CUDA;
    attr_set[dev] = true;
  }
  const int np = static_cast<int>(round_up(static_cast<size_t>(N), 128));
  const float scale_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
  // exponent factor of the main kernel: it subtracts LSE2 / c inside the score
  // GEMM, so c must not be 0; below 1e-30 every scaled score is 0 to fp32
  // accuracy anyway, and the exact scale is applied to dQ and dK afterwards
  const float c_exp = std::fabs(scale_log2) < 1e-30f ? (scale_log2 < 0.f ? -1e-30f : 1e-30f)
                                                     : scale_log2;
  {
    LaunchTimer timer(st, FA_KERNEL_BWD_PRE);
    const long long rows = static_cast<long long>(BH) * np;
    const long long rows_per_warp = 4LL * (32 / (D / 8));  // see bwd_preprocess_kernel
    const long long warps = (rows + rows_per_warp - 1) / rows_per_warp;
    // a grid-stride kernel: at most 8 blocks of 8 warps per SM
    const long long cap = 8LL * sm_count(dev);
    const unsigned blocks = static_cast<unsigned>(std::min((warps + 7) / 8, cap));
    fa::bwd_preprocess_kernel<D><<<blocks, 256, 0, st>>>(
        static_cast<const __nv_bfloat16*>(o), static_cast<const __nv_bfloat16*>(dout), lse,
        ws.dvec, ws.lse2, kDet ? nullptr : ws.dq_acc, BH, N, np,
        static_cast<float>(1.4426950408889634));
    if (cudaGetLastError() != cudaSuccess) return FA_ERR_CUDA;
  }
  {
    LaunchTimer timer(st, FA_KERNEL_BWD_MAIN);
    // work items (head, key tile); persistent: one CTA per SM, the kernel
    // maps item numbers to them
    const long long items = static_cast<long long>(BH) * (np / 128);
    if (items > 0x7fffffffLL) return FA_ERR_SHAPE;
    const int n_items = static_cast<int>(items);
    const int grid = std::min(n_items, sm_count(dev));
    const uint32_t slot = next_sched_slot(dev);
    fa::bwd_main_kernel<D, C, !kDet><<<grid, L::kThreads, L::kSmemAlloc, st>>>(
        mq, mk, mv, mdo, mdk, mdv, ws.dvec, ws.lse2, ws.dq_acc, N, np, scale, c_exp,
        kWaitLimitNs, BH, n_items, slot, bwd_head_group(BH, np, D));
    if (cudaGetLastError() != cudaSuccess) return FA_ERR_CUDA;
  }
  if (kDet) {
    LaunchTimer timer(st, FA_KERNEL_BWD_DQ);
    // one CTA per (head, Q tile), numbered in head groups whose K and V come
    // to about 32 MB, as the forward's
    const unsigned grid = static_cast<unsigned>(BH) * static_cast<unsigned>(np / 128);
    const long long kv_bytes = 4LL * np * D;
    const int hg = static_cast<int>(std::max(8LL, std::min(128LL, (32LL << 20) / kv_bytes)));
    fa::dq_pass_kernel<D, C><<<grid, LQ::kThreads, LQ::kSmemAlloc, st>>>(
        mq, mk, mv, mdo, mdq, ws.dvec, ws.lse2, N, np, scale, scale_log2, kWaitLimitNs, BH,
        std::min(hg, BH));
  } else {
    LaunchTimer timer(st, FA_KERNEL_BWD_DQ);
    const long long warps = (static_cast<long long>(BH) * N + 15) / 16 * (D / 16);
    const unsigned blocks = static_cast<unsigned>((warps + 7) / 8);  // 8 warps per block
    fa::dq_convert_kernel<D><<<blocks, 256, 0, st>>>(ws.dq_acc, static_cast<__nv_bfloat16*>(dq),
                                                      BH, N, np, scale);
  }
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

// Shared body of fa_bwd and fa_bwd_deterministic.
template <bool kDet>
fa_status bwd_entry(const void* q, const void* k, const void* v, const void* o, const float* lse,
                    const void* dout, void* dq, void* dk, void* dv, void* workspace,
                    size_t workspace_bytes, int B, int H, int N, int d, int causal, float scale,
                    void* stream) {
  if (!q || !k || !v || !o || !lse || !dout || !dq || !dk || !dv) return FA_ERR_NULL;
  fa_status st = check_common(B, H, N, d, scale);
  if (st != FA_OK) return st;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(dout) ||
      !aligned16(dq) || !aligned16(dk) || !aligned16(dv) ||
      (reinterpret_cast<uintptr_t>(lse) & 3u))
    return FA_ERR_ALIGN;
  const size_t need = bwd_workspace_layout(nullptr, B, H, N, d).bytes;
  if (!workspace || workspace_bytes < need) return FA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return FA_ERR_ALIGN;
  const int bh = B * H;
  BwdWorkspace ws = bwd_workspace_layout(workspace, B, H, N, d);
  CUtensorMap mq, mk, mv, mdo, mdk, mdv, mdq;
  if (!encode_bf16_3d(&mq, q, d, N, bh, 128) || !encode_bf16_3d(&mk, k, d, N, bh, 128) ||
      !encode_bf16_3d(&mv, v, d, N, bh, 128) || !encode_bf16_3d(&mdo, dout, d, N, bh, 128) ||
      !encode_out_box32(&mdk, dk, d, N, bh) || !encode_out_box32(&mdv, dv, d, N, bh) ||
      !encode_bf16_3d(&mdq, dq, d, N, bh, 128))
    return FA_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (d == 64)
    return causal ? launch_bwd<64, true, kDet>(mq, mk, mv, mdo, mdk, mdv, mdq, o, dout, lse, dq,
                                               ws, bh, N, scale, s)
                  : launch_bwd<64, false, kDet>(mq, mk, mv, mdo, mdk, mdv, mdq, o, dout, lse, dq,
                                                ws, bh, N, scale, s);
  return causal ? launch_bwd<128, true, kDet>(mq, mk, mv, mdo, mdk, mdv, mdq, o, dout, lse, dq,
                                              ws, bh, N, scale, s)
                : launch_bwd<128, false, kDet>(mq, mk, mv, mdo, mdk, mdv, mdq, o, dout, lse, dq,
                                               ws, bh, N, scale, s);
}

struct KvOuterWorkspace {
  float* o_acc;
  float* m;
  float* l;
  size_t bytes;
};

KvOuterWorkspace kv_outer_layout(void* base, int B, int H, int N, int d) {
  const size_t bh = static_cast<size_t>(B) * H;
  const size_t np = round_up(static_cast<size_t>(N), 128);
  const size_t acc = round_up(bh * np * d * sizeof(float), 256);
  const size_t vec = round_up(bh * np * sizeof(float), 256);
  char* p = static_cast<char*>(base);
  return {reinterpret_cast<float*>(p), reinterpret_cast<float*>(p + acc),
          reinterpret_cast<float*>(p + acc + vec), acc + 2 * vec};
}

template <int D, bool C>
fa_status launch_kv_outer(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                          const CUtensorMap& mo, float* lse, const KvOuterWorkspace& ws, int BH,
                          int N, float scale_log2, cudaStream_t st) {
  using L = fa::KvOuterLayout<D>;
  static bool attr_set[kMaxDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev >= kMaxDevices) return FA_ERR_CUDA;
  if (!attr_set[dev]) {
    if (!set_smem(fa::kv_outer_fwd_kernel<D, C>, L::kSmemAlloc)) return FA_ERR_CUDA;
    attr_set[dev] = true;
  }
  const int np = static_cast<int>(round_up(static_cast<size_t>(N), 128));
  {
    LaunchTimer timer(st, FA_KERNEL_FWD_KV_OUTER);
    fa::kv_outer_fwd_kernel<D, C><<<static_cast<unsigned>(BH), 256, L::kSmemAlloc, st>>>(
        mq, mk, mv, mo, lse, ws.o_acc, ws.m, ws.l, N, np, scale_log2, kWaitLimitNs);
  }
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

}  // namespace

extern "C" {

fa_status fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
                 int N, int d, int causal, float scale, void* stream) {
  if (!q || !k || !v || !o || !lse) return FA_ERR_NULL;
  fa_status st = check_common(B, H, N, d, scale);
  if (st != FA_OK) return st;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) ||
      (reinterpret_cast<uintptr_t>(lse) & 3u))
    return FA_ERR_ALIGN;
  const int bh = B * H;
  CUtensorMap mq, mk, mv, mo;
  if (!encode_bf16_3d(&mq, q, d, N, bh, 128) || !encode_bf16_3d(&mk, k, d, N, bh, 128) ||
      !encode_bf16_3d(&mv, v, d, N, bh, 128) || !encode_out_box32(&mo, o, d, N, bh))
    return FA_ERR_CUDA;
  const float scale_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (d == 64)
    return causal ? launch_fwd<64, true, false>(mq, mk, mv, mo, lse, bh, N, scale_log2, s)
                  : launch_fwd<64, false, false>(mq, mk, mv, mo, lse, bh, N, scale_log2, s);
  return causal ? launch_fwd<128, true, false>(mq, mk, mv, mo, lse, bh, N, scale_log2, s)
                : launch_fwd<128, false, false>(mq, mk, mv, mo, lse, bh, N, scale_log2, s);
}

size_t fa_fwd_splitkv_workspace_size(int B, int H, int N, int d, int num_splits) {
  if (check_common(B, H, N, d, 1.0f) != FA_OK) return 0;
  if (num_splits < 1 || num_splits > kMaxSplits) return 0;
  const size_t rows = static_cast<size_t>(num_splits) * B * H * round_up(static_cast<size_t>(N), 128);
  return rows * static_cast<size_t>(d + 1) * sizeof(float);  // partial O, then partial LSE
}

fa_status fa_fwd_splitkv(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                         int H, int N, int d, int causal, float scale, int num_splits,
                         void* workspace, size_t workspace_bytes, void* stream) {
  if (!q || !k || !v || !o || !lse) return FA_ERR_NULL;
  fa_status st = check_common(B, H, N, d, scale);
  if (st != FA_OK) return st;
  if (num_splits < 1 || num_splits > kMaxSplits) return FA_ERR_SHAPE;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) ||
      (reinterpret_cast<uintptr_t>(lse) & 3u))
    return FA_ERR_ALIGN;
  const size_t need = fa_fwd_splitkv_workspace_size(B, H, N, d, num_splits);
  if (!workspace || workspace_bytes < need) return FA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return FA_ERR_ALIGN;
  const int bh = B * H;
  CUtensorMap mq, mk, mv;
  if (!encode_bf16_3d(&mq, q, d, N, bh, 128) || !encode_bf16_3d(&mk, k, d, N, bh, 128) ||
      !encode_bf16_3d(&mv, v, d, N, bh, 128))
    return FA_ERR_CUDA;
  float* part_o = static_cast<float*>(workspace);
  float* part_lse =
      part_o + static_cast<size_t>(num_splits) * bh * round_up(static_cast<size_t>(N), 128) * d;
  const float scale_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  fa_status r;
  if (d == 64)
    r = causal ? launch_fwd<64, true, true>(mq, mk, mv, mq, lse, bh, N, scale_log2, s,
                                            num_splits, part_o, part_lse)
               : launch_fwd<64, false, true>(mq, mk, mv, mq, lse, bh, N, scale_log2, s,
                                             num_splits, part_o, part_lse);
  else
    r = causal ? launch_fwd<128, true, true>(mq, mk, mv, mq, lse, bh, N, scale_log2, s,
                                             num_splits, part_o, part_lse)
               : launch_fwd<128, false, true>(mq, mk, mv, mq, lse, bh, N, scale_log2, s,
                                              num_splits, part_o, part_lse);
  if (r != FA_OK) return r;
  {
    LaunchTimer timer(s, FA_KERNEL_FWD_COMBINE);
    const long long threads = static_cast<long long>(bh) * N * (d / 8);
    const unsigned blocks = static_cast<unsigned>((threads + 255) / 256);
    if (d == 64)
      fa::splitkv_combine_kernel<64><<<blocks, 256, 0, s>>>(
          part_o, part_lse, static_cast<__nv_bfloat16*>(o), lse, bh, N, num_splits);
    else
      fa::splitkv_combine_kernel<128><<<blocks, 256, 0, s>>>(
          part_o, part_lse, static_cast<__nv_bfloat16*>(o), lse, bh, N, num_splits);
  }
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

size_t fa_fwd_kv_outer_workspace_size(int B, int H, int N, int d) {
  if (check_common(B, H, N, d, 1.0f) != FA_OK) return 0;
  return kv_outer_layout(nullptr, B, H, N, d).bytes;
}

fa_status fa_fwd_kv_outer(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                          int H, int N, int d, int causal, float scale, void* workspace,
                          size_t workspace_bytes, void* stream) {
  if (!q || !k || !v || !o || !lse) return FA_ERR_NULL;
  fa_status st = check_common(B, H, N, d, scale);
  if (st != FA_OK) return st;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) ||
      (reinterpret_cast<uintptr_t>(lse) & 3u))
    return FA_ERR_ALIGN;
  const KvOuterWorkspace ws = kv_outer_layout(workspace, B, H, N, d);
  if (!workspace || workspace_bytes < ws.bytes) return FA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return FA_ERR_ALIGN;
  const int bh = B * H;
  CUtensorMap mq, mk, mv, mo;
  if (!encode_bf16_3d(&mq, q, d, N, bh, 128) || !encode_bf16_3d(&mk, k, d, N, bh, 128) ||
      !encode_bf16_3d(&mv, v, d, N, bh, 128) || !encode_bf16_3d(&mo, o, d, N, bh, 128))
    return FA_ERR_CUDA;
  const float scale_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (d == 64)
    return causal ? launch_kv_outer<64, true>(mq, mk, mv, mo, lse, ws, bh, N, scale_log2, s)
                  : launch_kv_outer<64, false>(mq, mk, mv, mo, lse, ws, bh, N, scale_log2, s);
  return causal ? launch_kv_outer<128, true>(mq, mk, mv, mo, lse, ws, bh, N, scale_log2, s)
                : launch_kv_outer<128, false>(mq, mk, mv, mo, lse, ws, bh, N, scale_log2, s);
}

size_t fa_bwd_workspace_size(int B, int H, int N, int d) {
  if (check_common(B, H, N, d, 1.0f) != FA_OK) return 0;
  return bwd_workspace_layout(nullptr, B, H, N, d).bytes;
}

fa_status fa_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse,
                 const void* dout, void* dq, void* dk, void* dv, void* workspace,
                 size_t workspace_bytes, int B, int H, int N, int d, int causal, float scale,
                 void* stream) {
  return bwd_entry<false>(q, k, v, o, lse, dout, dq, dk, dv, workspace, workspace_bytes, B, H, N,
                          d, causal, scale, stream);
}

fa_status fa_bwd_deterministic(const void* q, const void* k, const void* v, const void* o,
                               const float* lse, const void* dout, void* dq, void* dk, void* dv,
                               void* workspace, size_t workspace_bytes, int B, int H, int N,
                               int d, int causal, float scale, void* stream) {
  return bwd_entry<true>(q, k, v, o, lse, dout, dq, dk, dv, workspace, workspace_bytes, B, H, N,
                         d, causal, scale, stream);
}

}  // extern "C"

namespace {

// Scratch of fa_bwd_noalloc: one fixed device array per GPU, never allocated
// at call time.  Host code only ever sees its address through
// cudaGetSymbolAddress; the symbol itself is a host-side stand-in.
static __device__ __align__(256) unsigned char g_noalloc_scratch[FA_BWD_NOALLOC_SCRATCH_BYTES];

std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device (looked up once
// per device); nullptr if the lookup fails.
void* noalloc_scratch_address() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) return nullptr;
    g_noalloc_ptr[dev] = p;
  }
  return g_noalloc_ptr[dev];
}

}  // namespace

extern "C" {

fa_status fa_bwd_noalloc(const void* q, const void* k, const void* v, const void* o,
                         const float* lse, const void* dout, void* dq, void* dk, void* dv, int B,
                         int H, int N, int d, int causal, float scale, void* stream) {
  // same checks as fa_bwd, in the same order, before the scratch is touched
  if (!q || !k || !v || !o || !lse || !dout || !dq || !dk || !dv) return FA_ERR_NULL;
  fa_status st = check_common(B, H, N, d, scale);
  if (st != FA_OK) return st;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(dout) ||
      !aligned16(dq) || !aligned16(dk) || !aligned16(dv) ||
      (reinterpret_cast<uintptr_t>(lse) & 3u))
    return FA_ERR_ALIGN;
  const size_t need = bwd_workspace_layout(nullptr, B, H, N, d).bytes;
  if (need > FA_BWD_NOALLOC_SCRATCH_BYTES) return FA_ERR_WORKSPACE;
  void* scratch = noalloc_scratch_address();
  if (!scratch) return FA_ERR_CUDA;
  // the preprocess kernel rewrites every scratch word the main kernel reads
  // (the fp32 dQ accumulator is cleared, D and the log2 LSE are written)
  return fa_bwd(q, k, v, o, lse, dout, dq, dk, dv, scratch, FA_BWD_NOALLOC_SCRATCH_BYTES, B, H,
                N, d, causal, scale, stream);
}

fa_status fa_check_device_error(void* stream, unsigned int* detail) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return FA_ERR_CUDA;
  unsigned int word = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&word, fa::g_error_word, sizeof(word)) != cudaSuccess)
    return FA_ERR_CUDA;
  if (word && cudaMemcpyToSymbol(fa::g_error_word, &zero, sizeof(zero)) != cudaSuccess)
    return FA_ERR_CUDA;
  if (detail) *detail = word;
  return word ? FA_ERR_DEVICE_TIMEOUT : FA_OK;
}

fa_status fa_selftest_watchdog(unsigned int limit_ms, void* stream) {
  if (limit_ms < 1 || limit_ms > 2000) return FA_ERR_SHAPE;
  fa::watchdog_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<uint64_t>(limit_ms) * 1000000ull);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

const char* fa_status_string(fa_status s) {
  switch (s) {
    case FA_OK: return "ok";
    case FA_ERR_NULL: return "null pointer argument";
    case FA_ERR_SHAPE: return "invalid shape (B, H, N must be >= 1 and within limits)";
    case FA_ERR_UNSUPPORTED_D: return "unsupported head dimension (d must be 64 or 128)";
    case FA_ERR_ALIGN: return "tensor pointer not 16-byte aligned";
    case FA_ERR_SCALE: return "scale is not finite";
    case FA_ERR_WORKSPACE: return "workspace missing or too small";
    case FA_ERR_CUDA: return "CUDA runtime error";
    case FA_ERR_DEVICE_TIMEOUT: return "a kernel gave up on a bounded wait";
    case FA_ERR_STATE: return "timing calls out of order";
  }
  return "unknown status";
}

fa_status fa_timing_begin(void) {
  std::lock_guard<std::mutex> lock(g_timing.mu);
  if (g_timing.active) return FA_ERR_STATE;
  g_timing.active = true;
  return FA_OK;
}

fa_status fa_timing_end(float* ms_per_kernel, int* launches_per_kernel) {
  std::vector<TimedLaunch> done;
  {
    std::lock_guard<std::mutex> lock(g_timing.mu);
    if (!g_timing.active) return FA_ERR_STATE;
    g_timing.active = false;
    done.swap(g_timing.launches);
  }
  float ms[FA_KERNEL_COUNT] = {0};
  int cnt[FA_KERNEL_COUNT] = {0};
  fa_status st = FA_OK;
  for (auto& l : done) {
    float t = 0.f;
    if (cudaEventSynchronize(l.stop) != cudaSuccess ||
        cudaEventElapsedTime(&t, l.start, l.stop) != cudaSuccess)
      st = FA_ERR_CUDA;
    ms[l.kernel] += t;
    cnt[l.kernel] += 1;
  }
  {
    std::lock_guard<std::mutex> lock(g_timing.mu);
    for (auto& l : done) {
      g_timing.pool.push_back(l.start);
      g_timing.pool.push_back(l.stop);
    }
  }
  for (int i = 0; i < FA_KERNEL_COUNT; ++i) {
    if (ms_per_kernel) ms_per_kernel[i] = ms[i];
    if (launches_per_kernel) launches_per_kernel[i] = cnt[i];
  }
  return st;
}

int fa_version(void) { return 100; }

}  // extern "C"
