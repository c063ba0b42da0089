// Merge of the weighted routed expert outputs with the always-on shared
// expert(s) ("Model anatomy -- GLM-5.2", MoE panel: the renormalised, scaled
// expert outputs are merged with one always-on shared expert; "Expert fan-out
// 8 + 1").  Deterministic: each output element is summed in one fixed order,
// shared experts first, then slots 0..k-1, without atomics.  The output is
// fp32: a bf16 output could not stay within 2e-2 of the exact result once
// |out| >= 5.12, where half a bf16 ulp already exceeds 2e-2.
#include <cuda_bf16.h>

#include "moe_internal.cuh"
#include "sm100_ptx.cuh"

namespace moe {

constexpr int kCombineThreads = 256;
constexpr int kMaxK = 32;

// Block (t, c) merges columns [c * 2048, c * 2048 + 2048) of token t: each
// thread takes the float4 at column group v and then the one at v + 256, with
// the k + S row loads of each issued together.  Two column groups per thread
// keep the whole grid resident in one wave (at one group per thread the
// registers of a decode batch's 768 blocks need two).
constexpr int kCombineGroups = 2;

__global__ void __launch_bounds__(kCombineThreads) combine_kernel(
    const float* __restrict__ y, const float* __restrict__ w, const int32_t* __restrict__ inv,
    int T, int D, int k, int S, float* __restrict__ out, int* __restrict__ status,
    const int32_t* __restrict__ idx, uint32_t* __restrict__ mask, int mask_stride) {
  ptx::pdl_launch_dependents();
  ptx::pdl_wait();
  if (mask && blockIdx.y == 0 && threadIdx.x < k) {
    // this token's bit in the row of each expert it chose (set by the routing)
    const int t = blockIdx.x;
    const int e = idx[(size_t)t * k + threadIdx.x];
    if (e >= 0) atomicAnd(mask + (size_t)e * mask_stride + (t >> 5), ~(1u << (t & 31)));
  }
  __shared__ int s_row[kMaxK];
  __shared__ float s_w[kMaxK];
  const int t = blockIdx.x;
  const size_t rows_r = (size_t)T * k;
  if (threadIdx.x < k) {
    int r = inv[(size_t)t * k + threadIdx.x];
    if (r < 0 || (size_t)r >= rows_r) {
      if (status) atomicOr(status, kStBounds);
      r = -1;
    }
    s_row[threadIdx.x] = r;
    s_w[threadIdx.x] = w[(size_t)t * k + threadIdx.x];
  }
  __syncthreads();
#pragma unroll 1
  for (int g = 0; g < kCombineGroups; ++g) {
    const int v = (blockIdx.y * kCombineGroups + g) * kCombineThreads + threadIdx.x;
    if (v >= D / 4) break;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    // the first shared row is loaded with the first batch of routed rows, so a
    // layer with one shared expert and k <= 8 reads all its rows in one round
    float4 sh0 = make_float4(0.f, 0.f, 0.f, 0.f);
    if (S > 0) sh0 = reinterpret_cast<const float4*>(y + (rows_r + t) * D)[v];
    for (int j0 = 0; j0 < k; j0 += 8) {
      float4 a[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const int r = (j0 + q < k) ? s_row[j0 + q] : -1;
        a[q] = r >= 0 ? reinterpret_cast<const float4*>(y + (size_t)r * D)[v]
                      : make_float4(0.f, 0.f, 0.f, 0.f);
      }
      if (j0 == 0) {
        // shared experts first, in order
        acc.x += sh0.x; acc.y += sh0.y; acc.z += sh0.z; acc.w += sh0.w;
        for (int s = 1; s < S; ++s) {
          const float4 b = reinterpret_cast<const float4*>(y + (rows_r + (size_t)s * T + t) * D)[v];
          acc.x += b.x; acc.y += b.y; acc.z += b.z; acc.w += b.w;
        }
      }
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        if (j0 + q >= k || s_row[j0 + q] < 0) continue;
        const float wj = s_w[j0 + q];
        acc.x = fmaf(wj, a[q].x, acc.x);
        acc.y = fmaf(wj, a[q].y, acc.y);
        acc.z = fmaf(wj, a[q].z, acc.z);
        acc.w = fmaf(wj, a[q].w, acc.w);
      }
    }
    reinterpret_cast<float4*>(out + (size_t)t * D)[v] = acc;
  }
}

cudaError_t launch_combine(const float* y, const float* w, const int32_t* inv, int T, int D,
                           int k, int S, float* out, int* status, const int32_t* idx,
                           uint32_t* mask, int mask_stride, cudaStream_t st) {
  if (T == 0) return cudaSuccess;
  const int per_block = kCombineThreads * kCombineGroups;   // float4 column groups
  const dim3 grid(T, (D / 4 + per_block - 1) / per_block);
  return launch_pdl(combine_kernel, grid, dim3(kCombineThreads), 0, st, y, w, inv, T, D, k, S, out,
                    status, idx, mask, mask_stride);
}

}  // namespace moe
