// Router logits and routing.
//
// Router logits: the learned fp32 router ("Model anatomy -- GLM-5.2",
// Feed-forward / Mixture of Experts panel, "Routing: learned").  Small batches
// split the hidden dimension into partial sums so that every SM streams a
// distinct slice of the router weight; the partials are added in a fixed
// order by the consumer (routing kernel or the reduce kernel), so the logits
// are bit-reproducible.
//
// Routing (same panel): sigmoid router scores; the correction bias is added
// for the top-k selection only; the selected un-biased scores are
// renormalised and scaled by the routed scaling factor.  One warp per token,
// top-k by warp-shuffle arg-max rounds.
#include <cuda_bf16.h>

#include <cfloat>
#include <climits>

#include "moe_internal.cuh"

namespace moe {

RouterSplit router_split(int T, int D, int E) {
  const int tiles = ((T + kRouterTileT - 1) / kRouterTileT) * ((E + kRouterTileE - 1) / kRouterTileE);
  int want = (kSplitTargetBlocks + tiles - 1) / (tiles > 0 ? tiles : 1);
  if (want < 1) want = 1;
  if (want > 32) want = 32;
  int chunk = (D + want - 1) / want;
  chunk = (chunk + kRouterTileD - 1) / kRouterTileD * kRouterTileD;
  RouterSplit sp;
  sp.chunk = chunk;
  sp.nsplit = (D + chunk - 1) / chunk;
  return sp;
}

// out[s][t][e] = sum over d in split s of h[t, d] * Wr[e, d], d ascending.
// 256 threads; each owns a 4 (tokens) x 4 (experts) block of the 64 x 64 tile.
__global__ void __launch_bounds__(256) router_partials_kernel(const uint16_t* __restrict__ h,
                                                              const float* __restrict__ Wr,
                                                              int T, int D, int E, int chunk,
                                                              float* __restrict__ out) {
  __shared__ __align__(16) float hs[kRouterTileD][kRouterTileT + 4];
  __shared__ __align__(16) float wsm[kRouterTileD][kRouterTileE + 4];
  const int tid = threadIdx.x;
  const int e0 = blockIdx.x * kRouterTileE;
  const int t0 = blockIdx.y * kRouterTileT;
  const int s = blockIdx.z;
  const int dbeg = s * chunk;
  const int dend = min(D, dbeg + chunk);
  const int tx = tid & 15, ty = tid >> 4;

  float acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;

  const int lrow = tid >> 2;          // 0..63: token (h tile) / expert (Wr tile)
  const int lcol = (tid & 3) * 8;     // 0, 8, 16, 24 within the 32-wide d slice
  for (int d0 = dbeg; d0 < dend; d0 += kRouterTileD) {
    {
      const int t = t0 + lrow, d = d0 + lcol;
      float v[8];
      if (t < T && d < dend) {
        const uint4 raw = *reinterpret_cast<const uint4*>(h + (size_t)t * D + d);
        const uint32_t u[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          v[2 * i] = __uint_as_float(u[i] << 16);
          v[2 * i + 1] = __uint_as_float(u[i] & 0xFFFF0000u);
        }
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) v[i] = 0.f;
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) hs[lcol + i][lrow] = v[i];
    }
    {
      const int e = e0 + lrow, d = d0 + lcol;
      float v[8];
      if (e < E && d < dend) {
        const float4 a = *reinterpret_cast<const float4*>(Wr + (size_t)e * D + d);
        const float4 b = *reinterpret_cast<const float4*>(Wr + (size_t)e * D + d + 4);
        v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
        v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) v[i] = 0.f;
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) wsm[lcol + i][lrow] = v[i];
    }
    __syncthreads();
#pragma unroll 8
    for (int kk = 0; kk < kRouterTileD; ++kk) {
      const float4 a = *reinterpret_cast<const float4*>(&hs[kk][ty * 4]);
      const float4 b = *reinterpret_cast<const float4*>(&wsm[kk][tx * 4]);
      const float av[4] = {a.x, a.y, a.z, a.w};
      const float bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
    }
    __syncthreads();
  }
  float* o = out + (size_t)s * T * E;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int t = t0 + ty * 4 + i;
    if (t >= T) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int e = e0 + tx * 4 + j;
      if (e < E) o[(size_t)t * E + e] = acc[i][j];
    }
  }
}

__global__ void reduce_partials_kernel(const float* __restrict__ p, int nsplit, size_t n,
                                       float* __restrict__ out) {
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n;
       i += (size_t)gridDim.x * blockDim.x) {
    float v = p[i];
    for (int s = 1; s < nsplit; ++s) v = __fadd_rn(v, p[(size_t)s * n + i]);
    out[i] = v;
  }
}

cudaError_t launch_router_partials(const uint16_t* h, const float* Wr, int T, int D, int E,
                                   RouterSplit sp, float* out, cudaStream_t st) {
  dim3 grid((E + kRouterTileE - 1) / kRouterTileE, (T + kRouterTileT - 1) / kRouterTileT,
            sp.nsplit);
  router_partials_kernel<<<grid, 256, 0, st>>>(h, Wr, T, D, E, sp.chunk, out);
  return cudaGetLastError();
}

cudaError_t launch_reduce_partials(const float* partials, int nsplit, size_t n, float* out,
                                   cudaStream_t st) {
  const int threads = 256;
  size_t blocks = (n + threads - 1) / threads;
  if (blocks > 4096) blocks = 4096;
  if (blocks == 0) return cudaSuccess;
  reduce_partials_kernel<<<(unsigned)blocks, threads, 0, st>>>(partials, nsplit, n, out);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// routing
// ---------------------------------------------------------------------------
constexpr int kRouteWarps = 4;

// (key, expert) pair a precedes b under (key descending, index ascending).
__device__ __forceinline__ bool precedes(float ka, int ea, float kb, int eb) {
  return ka > kb || (ka == kb && ea < eb);
}

template <int EPL>
__global__ void __launch_bounds__(kRouteWarps * 32) route_kernel(
    const float* __restrict__ src, int nsplit, const float* __restrict__ bias, int T, int E,
    int k, float scale, int32_t* __restrict__ idx, float* __restrict__ w,
    int* __restrict__ status) {
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * kRouteWarps + (threadIdx.x >> 5);
  if (t >= T) return;
  const size_t plane = (size_t)T * E;

  float key[EPL], sc[EPL];
  bool bad = false;
#pragma unroll
  for (int i = 0; i < EPL; ++i) {
    const int e = lane + 32 * i;
    if (e < E) {
      float l = src[(size_t)t * E + e];
      for (int s = 1; s < nsplit; ++s) l = __fadd_rn(l, src[s * plane + (size_t)t * E + e]);
      // sigmoid in fp64 from the fp32 logit, rounded once to fp32
      const double sd = 1.0 / (1.0 + exp(-(double)l));
      sc[i] = __double2float_rn(sd);
      key[i] = __fadd_rn(sc[i], bias[e]);
      if (!isfinite(l) || !isfinite(key[i])) bad = true;
    } else {
      sc[i] = 0.f;
      key[i] = -FLT_MAX;
    }
  }
  if (__any_sync(0xffffffffu, bad)) {
    if (lane == 0 && status) atomicOr(status, kStNonFinite);
  }

  unsigned taken = 0u;          // bit i: expert lane + 32 i already selected
  int my_e = 0;                 // slot `lane`'s expert (lanes < k)
  float my_s = 0.f;             // and its un-biased score
  float sum = 0.f;
  for (int j = 0; j < k; ++j) {
    float bk = -INFINITY;
    int be = INT_MAX;
    float bs = 0.f;
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
      const int e = lane + 32 * i;
      if (e < E && !(taken & (1u << i)) && precedes(key[i], e, bk, be)) {
        bk = key[i];
        be = e;
        bs = sc[i];
      }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      const float ok = __shfl_xor_sync(0xffffffffu, bk, off);
      const int oe = __shfl_xor_sync(0xffffffffu, be, off);
      const float os = __shfl_xor_sync(0xffffffffu, bs, off);
      if (precedes(ok, oe, bk, be)) {
        bk = ok;
        be = oe;
        bs = os;
      }
    }
    if (be != INT_MAX && (be & 31) == lane) taken |= 1u << (be >> 5);
    if (lane == j) {
      my_e = be;
      my_s = bs;
    }
    sum = (j == 0) ? bs : __fadd_rn(sum, bs);
  }
  if (lane < k) {
    idx[(size_t)t * k + lane] = my_e;
    w[(size_t)t * k + lane] = __fmul_rn(__fdiv_rn(my_s, sum), scale);
  }
}

cudaError_t launch_route(const float* src, int nsplit, const float* bias, int T, int E, int k,
                         float scale, int32_t* idx, float* w, int* status, cudaStream_t st) {
  const dim3 grid((T + kRouteWarps - 1) / kRouteWarps);
  const dim3 block(kRouteWarps * 32);
  const int epl = (E + 31) / 32;
  if (epl <= 1)
    route_kernel<1><<<grid, block, 0, st>>>(src, nsplit, bias, T, E, k, scale, idx, w, status);
  else if (epl <= 2)
    route_kernel<2><<<grid, block, 0, st>>>(src, nsplit, bias, T, E, k, scale, idx, w, status);
  else if (epl <= 4)
    route_kernel<4><<<grid, block, 0, st>>>(src, nsplit, bias, T, E, k, scale, idx, w, status);
  else if (epl <= 8)
    route_kernel<8><<<grid, block, 0, st>>>(src, nsplit, bias, T, E, k, scale, idx, w, status);
  else if (epl <= 16)
    route_kernel<16><<<grid, block, 0, st>>>(src, nsplit, bias, T, E, k, scale, idx, w, status);
  else
    route_kernel<32><<<grid, block, 0, st>>>(src, nsplit, bias, T, E, k, scale, idx, w, status);
  return cudaGetLastError();
}

}  // namespace moe
