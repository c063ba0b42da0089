// Internal declarations shared by the library's translation units.
#pragma once

#include <atomic>

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>
#include <utility>

#include "../../include/moe_b200.h"

namespace moe {

// Bits of the device status word (first int32 of the workspace).
constexpr int kStNonFinite = 1;
constexpr int kStBounds = 2;
constexpr int kStTimeout = 4;

// Block count a small problem is split into (one wave on the 148 SMs of a
// B200); the split depends on the shape only, so results are bit-identical
// on every device.
constexpr int kSplitTargetBlocks = 148;

// Router logits tiling (fp32 FMA, split over D).
constexpr int kRouterTileT = 64;
constexpr int kRouterTileE = 64;
constexpr int kRouterTileD = 32;

// How the router logits are computed: on the tensor cores (three-way bf16
// split of the router weight, needs D % 64 == 0 and E % 8 == 0) or with fp32
// FMAs; both produce `nsplit` partial-sum planes [T, E] added in order.
struct RouterSplit {
  bool tensor;  // tensor-core path
  bool fused;   // tensor-core path that splits the fp32 weight in the kernel
  int nsplit;   // partial-sum planes
  int chunk;    // reduction range of one plane (over D for FMA and fused, over 3D for tensor)
};
// The fused tensor-core router (router_tc.cu): batches of at most
// kRouterTcMaxT tokens with D % 64 == 0 and E % 32 == 0.
constexpr int kRouterTcMaxT = 256;
bool router_tc_shape_ok(int T, int D, int E);
void router_tc_split(int T, int D, int E, int* nsplit, int* kb_per);
cudaError_t launch_router_tc_fused(const uint16_t* h, const float* Wr, int T, int D, int E,
                                   int nsplit, int kb_per, float* partials, int* status,
                                   cudaStream_t st, const char** why);
RouterSplit router_split(int T, int D, int E);
int router_tile_n(int T, int E);  // MMA N of the tensor-core router

// Permute: tokens per counting block.
constexpr int kPermBlockTokens = 256;
// Capacity of the grouping's static scratch (allocation-free variant):
// 64 counting blocks (T <= 16384) x 1024 experts, 256 KiB.
constexpr int kNoAllocMaxBlocks = 64;
constexpr int kNoAllocMaxExperts = 1024;
cudaError_t noalloc_scratch(int32_t** out);

// Workspace layout (byte offsets from the workspace base, 256-aligned).
struct WsLayout {
  size_t status, ticket, partials, wr3, idx, w, counts, offsets, perm, inv, blk_base, counters,
      counters_s, xperm,
      act_r, act_s, y, touched, gmask, total;
};
bool ws_layout(const moe_dims_t& d, WsLayout* out);

// Raises a kernel's dynamic shared-memory limit to `bytes` on the current
// device, once per device: `done` holds one bit per device ordinal (two host
// threads that race on a device's first call both set the attribute, which
// is harmless).
template <typename Kernel>
cudaError_t set_smem_once(Kernel kernel, int bytes, std::atomic<uint64_t>& done) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t bit = 1ull << (dev & 63);
  if (done.load(std::memory_order_acquire) & bit) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess) done.fetch_or(bit, std::memory_order_release);
  return e;
}

// Launch with programmatic dependent launch allowed: the kernel may start
// while the previous kernel in the stream finishes; every kernel of the
// library waits (griddepcontrol.wait) before it reads what earlier kernels
// wrote, and lets its successor launch as soon as it starts.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t st, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// --- launchers (return cudaSuccess or the launch error) ---------------------
cudaError_t launch_router_partials(const uint16_t* h, const float* Wr, int T, int D, int E,
                                   RouterSplit sp, float* out, cudaStream_t st);
cudaError_t launch_split_router(const float* Wr, int E, int D, uint16_t* wr3, cudaStream_t st);
cudaError_t launch_router_tc(const uint16_t* h, const uint16_t* wr3, int T, int D, int E,
                             int nsplit, int chunk, float* partials, cudaStream_t st,
                             const char** why);
cudaError_t launch_reduce_partials(const float* partials, int nsplit, size_t n, float* out,
                                   cudaStream_t st);
cudaError_t launch_route(const float* src, int nsplit, const float* bias, int T, int E, int k,
                         float scale, int32_t* idx, float* w, int* status, cudaStream_t st);
// Outputs of the grouping done by the routing kernel's last block (as
// launch_permute's); `ticket` is an int that is zero before the launch and
// is left zero after it.
struct RouteGrouping {
  int32_t* counts;
  int32_t* offsets;
  int32_t* perm;
  int32_t* inv;
  int32_t* touched;
  int* ticket;  // nullptr: no grouping
  // [E][kPermBlockTokens / 32] token bitmask per expert, zero between calls:
  // each token's block sets its bits, the last block reads and clears them
  uint32_t* mask;
};
// Routing that also sets token t's bit in row idx[t, j] of `mask`
// [E][kPermBlockTokens / 32] (zero on entry) for every slot j; T <= kPermBlockTokens.
cudaError_t launch_route_bits(const float* src, int nsplit, const float* bias, int T, int E,
                              int k, float scale, int32_t* idx, float* w, int* status,
                              uint32_t* mask, cudaStream_t st);
// Routing and grouping in one launch; T <= kPermBlockTokens.
cudaError_t launch_route_and_group(const float* src, int nsplit, const float* bias, int T, int E,
                                   int k, float scale, int32_t* idx, float* w, int* status,
                                   const RouteGrouping& grp, cudaStream_t st);
// `touched` (nullable): number of experts with at least one pair.
cudaError_t launch_route_grouped(const float* logits, const float* bias, int T, int E, int k,
                                 float scale, int n_group, int topk_group, int32_t* idx, float* w,
                                 int* status, cudaStream_t st);
cudaError_t launch_permute(const int32_t* idx, int T, int E, int k, int32_t* counts,
                           int32_t* offsets, int32_t* perm, int32_t* inv, int32_t* blk_base,
                           int* status, int32_t* touched, cudaStream_t st, int* nlaunch);
// Also zeroes the expert FFN's per-group counters and tile claim counter
// (`ncounters` ints).
cudaError_t launch_gather_rows(const uint16_t* h, const int32_t* perm, int rows, int D, int T,
                               uint16_t* xperm, int* counters, int ncounters, cudaStream_t st);
// With `mask` set, the blocks of column chunk 0 also clear every token's bits
// in the rows [E][mask_stride] of the experts idx names (the routing set them).
cudaError_t launch_combine(const float* y, const float* w, const int32_t* inv, int T, int D,
                           int k, int S, float* out, int* status, const int32_t* idx,
                           uint32_t* mask, int mask_stride, cudaStream_t st);

// Expert MLPs: gate/up GEMM with the SiLU gate fused, then the down GEMM.
struct FfnArgs {
  const uint16_t* xperm;    // [T*k, D] gathered routed rows
  const uint16_t* h;        // [T, D] (A operand of the shared experts)
  const int32_t* offsets;   // [E+1]
  const uint16_t *W1, *W3, *W2, *Ws1, *Ws3, *Ws2;
  uint16_t* act_r;          // [T*k, F]
  uint16_t* act_s;          // [S*T, Fs]
  float* y;                 // [T*k + S*T, D]
  int* status;
  int* counters;            // [E + S + 1], zero at launch (group counters, tile claims)
  int T, D, E, F, k, S, Fs;
  // Which groups one launch runs: all, the routed experts only, or the shared
  // experts only (then `counters_s` [S + 2] holds their group counters, tile
  // claims and an exit ticket; zero at launch, and the launch's last CTA to
  // finish zeroes them again; the grid is at most `max_ctas` CTAs).
  int part = 0;
  int* counters_s = nullptr;
  int max_ctas = 0;
  // dense_a batches routed without a grouping pass (GemmParams::mask)
  const uint32_t* mask = nullptr;
  int mask_stride = 0;
  int32_t* counts_out = nullptr;
  int32_t* offsets_out = nullptr;
  int32_t* touched_out = nullptr;
  int32_t* inv_out = nullptr;
  // 1: the launch's last CTA zeroes `counters` (E + S group counters, the
  // claim counter and the exit ticket at [E + S + 1]) itself
  int self_reset = 0;
  // T <= kDenseMaxT with bf16 weights: the routed gate/up A operand is h
  // itself (xperm is not used) and rows are placed by idx / inv [T, k].
  int dense_a = 0;
  const int32_t* idx = nullptr;
  const int32_t* inv = nullptr;
};
constexpr int kDenseMaxT = 128;
constexpr int kFfnAll = 0, kFfnRouted = 1, kFfnShared = 2;
// Batches of at most this many tokens run the shared experts (bf16 weights of
// at least kOverlapSharedMinBytes) on an internal stream, next to the routing,
// on at most kSharedCtas SMs.
constexpr int kOverlapSharedMaxT = 512;
constexpr double kOverlapSharedMinBytes = 16.0 * 1024 * 1024;
constexpr int kSharedCtas = 32;
// `marks` (nullable): one event recorded after the expert FFN kernel.
cudaError_t launch_expert_ffn(const FfnArgs& a, cudaStream_t st, int* nlaunch,
                              const char** why, void* const* marks);

// FP8 expert weights: E4M3 codes and int8 block exponents (one per 128 x 128
// block of each expert's [rows, K] matrix).
struct Fp8Weights {
  const uint8_t *W1, *W3, *W2, *Ws1, *Ws3, *Ws2;
  const int8_t *W1e, *W3e, *W2e, *Ws1e, *Ws3e, *Ws2e;
};
// The expert MLPs of FfnArgs (whose bf16 weight pointers are unused) with FP8
// weights.
cudaError_t launch_expert_ffn_fp8(const FfnArgs& a, const Fp8Weights& w, cudaStream_t st,
                                  int* nlaunch, const char** why, void* const* marks);
// codes [G, R, K] + exps [G, ceil(R/128), ceil(K/128)] -> bf16 [G, R, K]; K % 16 == 0.
cudaError_t launch_fp8_dequantize(const uint8_t* codes, const int8_t* exps, int G, int R, int K,
                                  uint16_t* out, int* status, cudaStream_t st);

// dst[i] = src[idx[i]] for n rows of row_bytes (a multiple of 16) bytes.
cudaError_t launch_gather_bytes(const void* src, int src_rows, const int32_t* idx, int n,
                                int row_bytes, void* dst, int* status, cudaStream_t st);

int num_sms();

cudaError_t launch_bounded_wait_selftest(int* status, cudaStream_t st);
cudaError_t launch_occupy_selftest(int nctas, long long cycles, cudaStream_t st);

}  // namespace moe
