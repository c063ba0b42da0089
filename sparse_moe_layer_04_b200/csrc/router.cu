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
#include "permute_block.cuh"
#include "sm100_ptx.cuh"

namespace moe {

int router_tile_n(int T, int E) { return (E <= 128 || T <= 512) ? 128 : 256; }

RouterSplit router_split(int T, int D, int E) {
  RouterSplit sp;
  sp.fused = false;
  if (router_tc_shape_ok(T, D, E)) {
    int kb_per = 1;
    sp.tensor = true;
    sp.fused = true;
    router_tc_split(T, D, E, &sp.nsplit, &kb_per);
    sp.chunk = kb_per * 64;
    return sp;
  }
  if (D % 64 == 0 && E % 8 == 0) {
    // tensor path: enough (row tile, column tile, K' chunk) work units for
    // about one wave; at most 64 planes
    const int kblocks = 3 * D / 64;
    const int bn = router_tile_n(T, E);
    const int tiles = ((T + 127) / 128) * ((E + bn - 1) / bn);
    int want = kSplitTargetBlocks / (tiles > 0 ? tiles : 1);  // at most one wave
    want = want < 1 ? 1 : (want > 64 ? 64 : want);
    const int kb_per = (kblocks + want - 1) / want;
    sp.tensor = true;
    sp.chunk = kb_per * 64;
    sp.nsplit = (kblocks + kb_per - 1) / kb_per;
    return sp;
  }
  const int tiles = ((T + kRouterTileT - 1) / kRouterTileT) * ((E + kRouterTileE - 1) / kRouterTileE);
  int want = (kSplitTargetBlocks + tiles - 1) / (tiles > 0 ? tiles : 1);
  if (want < 1) want = 1;
  if (want > 32) want = 32;
  int chunk = (D + want - 1) / want;
  chunk = (chunk + kRouterTileD - 1) / kRouterTileD * kRouterTileD;
  sp.tensor = false;
  sp.chunk = chunk;
  sp.nsplit = (D + chunk - 1) / chunk;
  return sp;
}

// wr3[e] = [hi | mid | lo] with hi = bf16(w), mid = bf16(w - hi),
// lo = bf16(w - hi - mid); both subtractions are exact (Sterbenz), and each
// bf16 rounding leaves at most 2^-8 of what it rounds, so
// |w - (hi + mid + lo)| <= 2^-24 |w|: the fp32 value to within its own
// rounding.
__global__ void split_router_kernel(const float* __restrict__ Wr, int E, int D,
                                    uint16_t* __restrict__ wr3) {
  ptx::pdl_launch_dependents();
  ptx::pdl_wait();
  const size_t n4 = (size_t)E * D / 4;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n4;
       i += (size_t)gridDim.x * blockDim.x) {
    const float4 w = reinterpret_cast<const float4*>(Wr)[i];
    const size_t flat = i * 4;
    const size_t e = flat / D, d = flat % D;
    const float wv[4] = {w.x, w.y, w.z, w.w};
    uint16_t hi[4], mid[4], lo[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const __nv_bfloat16 bh = __float2bfloat16_rn(wv[q]);
      const float r1 = __fsub_rn(wv[q], __bfloat162float(bh));
      const __nv_bfloat16 bm = __float2bfloat16_rn(r1);
      const float r2 = __fsub_rn(r1, __bfloat162float(bm));
      const __nv_bfloat16 bl = __float2bfloat16_rn(r2);
      hi[q] = __bfloat16_as_ushort(bh);
      mid[q] = __bfloat16_as_ushort(bm);
      lo[q] = __bfloat16_as_ushort(bl);
    }
    uint16_t* row = wr3 + e * 3 * (size_t)D;
    *reinterpret_cast<uint2*>(row + d) =
        make_uint2(hi[0] | ((uint32_t)hi[1] << 16), hi[2] | ((uint32_t)hi[3] << 16));
    *reinterpret_cast<uint2*>(row + D + d) =
        make_uint2(mid[0] | ((uint32_t)mid[1] << 16), mid[2] | ((uint32_t)mid[3] << 16));
    *reinterpret_cast<uint2*>(row + 2 * (size_t)D + d) =
        make_uint2(lo[0] | ((uint32_t)lo[1] << 16), lo[2] | ((uint32_t)lo[3] << 16));
  }
}

cudaError_t launch_split_router(const float* Wr, int E, int D, uint16_t* wr3, cudaStream_t st) {
  const size_t n4 = (size_t)E * D / 4;
  size_t blocks = (n4 + 255) / 256;
  if (blocks > 2048) blocks = 2048;
  return launch_pdl(split_router_kernel, dim3((unsigned)blocks), dim3(256), 0, st, Wr, E, D, wr3);
}

// out[s][t][e] = sum over d in split s of h[t, d] * Wr[e, d], d ascending.
// 256 threads; each owns a 4 (tokens) x 4 (experts) block of the 64 x 64 tile.
__global__ void __launch_bounds__(256) router_partials_kernel(const uint16_t* __restrict__ h,
                                                              const float* __restrict__ Wr,
                                                              int T, int D, int E, int chunk,
                                                              float* __restrict__ out) {
  ptx::pdl_launch_dependents();
  ptx::pdl_wait();
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
  const int t_ld = t0 + lrow, e_ld = e0 + lrow;
  uint4 hraw = make_uint4(0, 0, 0, 0);
  float4 wa = make_float4(0.f, 0.f, 0.f, 0.f), wb = wa;
  // global -> registers for the slice at d0 (zeros outside the tensor)
  auto fetch = [&](int d0) {
    const int d = d0 + lcol;
    hraw = make_uint4(0, 0, 0, 0);
    wa = wb = make_float4(0.f, 0.f, 0.f, 0.f);
    if (d < dend) {
      if (t_ld < T) hraw = *reinterpret_cast<const uint4*>(h + (size_t)t_ld * D + d);
      if (e_ld < E) {
        wa = *reinterpret_cast<const float4*>(Wr + (size_t)e_ld * D + d);
        wb = *reinterpret_cast<const float4*>(Wr + (size_t)e_ld * D + d + 4);
      }
    }
  };
  if (dbeg < dend) fetch(dbeg);
  for (int d0 = dbeg; d0 < dend; d0 += kRouterTileD) {
    {
      const uint32_t u[4] = {hraw.x, hraw.y, hraw.z, hraw.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        hs[lcol + 2 * i][lrow] = __uint_as_float(u[i] << 16);
        hs[lcol + 2 * i + 1][lrow] = __uint_as_float(u[i] & 0xFFFF0000u);
      }
      const float v[8] = {wa.x, wa.y, wa.z, wa.w, wb.x, wb.y, wb.z, wb.w};
#pragma unroll
      for (int i = 0; i < 8; ++i) wsm[lcol + i][lrow] = v[i];
    }
    __syncthreads();
    if (d0 + kRouterTileD < dend) fetch(d0 + kRouterTileD);  // in flight during the FMAs
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
  ptx::pdl_launch_dependents();
  ptx::pdl_wait();
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
  return launch_pdl(router_partials_kernel, grid, dim3(256), 0, st, h, Wr, T, D, E, sp.chunk, out);
}

cudaError_t launch_reduce_partials(const float* partials, int nsplit, size_t n, float* out,
                                   cudaStream_t st) {
  const int threads = 256;
  size_t blocks = (n + threads - 1) / threads;
  if (blocks > 4096) blocks = 4096;
  if (blocks == 0) return cudaSuccess;
  return launch_pdl(reduce_partials_kernel, dim3((unsigned)blocks), dim3(threads), 0, st, partials,
                    nsplit, n, out);
}

// ---------------------------------------------------------------------------
// routing: one block per token, one thread per expert
// ---------------------------------------------------------------------------
// Selection order: key descending, then expert index ascending.  A key is
// mapped to an unsigned integer that orders the same way (-0 as +0; NaN, and
// "no candidate", as 0, below every key), so one warp-wide max reduction
// finds the best key and one min reduction over the lanes holding it the
// lowest expert index.
__device__ __forceinline__ uint32_t key_order(float key) {
  uint32_t u = __float_as_uint(key);
  if (key != key) return 0u;
  if (u == 0x80000000u) u = 0u;  // -0 ranks as +0
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Best (order, expert) pair of the warp; every lane gets the winner.
__device__ __forceinline__ void warp_best(uint32_t& bu, int& be) {
  const uint32_t m = __reduce_max_sync(0xffffffffu, bu);
  const uint32_t e = __reduce_min_sync(0xffffffffu, bu == m ? (uint32_t)be : 0xffffffffu);
  bu = m;
  be = (int)e;
}

constexpr int kMaxSlots = 32;

// Top-k of one token held one expert per thread (key, score, index; threads
// past E hold index INT_MAX), in the block's shared candidate arrays: each
// warp extracts its k best (key, index) pairs by warp arg-max rounds; the
// union of the warps' lists holds the token's top k, which warp 0 extracts
// the same way, in selection order, and writes with the renormalised weights
// (un-biased scores, fp32 sum in slot order, one division and one multiply).
// Must be called by every thread of the block.
__device__ __forceinline__ void block_topk_write(float key, float sc, int me, int t, int k,
                                                 float scale, int32_t* __restrict__ idx,
                                                 float* __restrict__ w, uint32_t* c_u, int* c_e,
                                                 float* s_sc) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = blockDim.x >> 5;
  uint32_t u = me != INT_MAX ? key_order(key) : 0u;
  if (me != INT_MAX) s_sc[me] = sc;
  for (int j = 0; j < k; ++j) {
    uint32_t bu = u;
    int be = me;
    warp_best(bu, be);
    if (lane == 0) {
      c_u[wid * k + j] = bu;
      c_e[wid * k + j] = bu ? be : INT_MAX;
    }
    if (be == me) u = 0u;
  }
  __syncthreads();
  if (wid != 0) return;
  const int nc = nw * k;
  unsigned done = 0u;  // bit q: candidate lane + 32 q already selected
  int my_e = 0;
  float my_s = 0.f, sum = 0.f;
  for (int j = 0; j < k; ++j) {
    uint32_t bu = 0u;
    int be = INT_MAX, bq = -1;
    for (int q = 0, c = lane; c < nc; ++q, c += 32) {
      if ((done >> q) & 1u) continue;
      const uint32_t cu = c_u[c];
      const int ce = c_e[c];
      if (ce != INT_MAX && (cu > bu || (cu == bu && ce < be))) {
        bu = cu;
        be = ce;
        bq = q;
      }
    }
    const int mine = be;
    warp_best(bu, be);
    if (bq >= 0 && mine == be) done |= 1u << bq;
    const float bs = be != INT_MAX ? s_sc[be] : 0.f;
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

// Sum of expert e's logit planes in plane order, its sigmoid (fp64, rounded
// once to fp32) and its selection key.  Returns false for a non-finite value.
__device__ __forceinline__ bool score_and_key(const float* __restrict__ src, int nsplit,
                                              size_t plane, size_t at, float b, float* sc,
                                              float* key) {
  const float* p = src + at;
  float l = p[0];
  // up to 32 plane loads in flight at once (the tensor-core router writes up
  // to 64 planes); the sum still runs in plane order
  for (int s0 = 1; s0 < nsplit; s0 += 32) {
    float v[32];
#pragma unroll
    for (int q = 0; q < 32; ++q) v[q] = (s0 + q < nsplit) ? p[(s0 + q) * plane] : 0.f;
#pragma unroll
    for (int q = 0; q < 32; ++q)
      if (s0 + q < nsplit) l = __fadd_rn(l, v[q]);
  }
  const double sd = 1.0 / (1.0 + exp(-(double)l));
  *sc = __double2float_rn(sd);
  *key = __fadd_rn(*sc, b);
  return isfinite(l) && isfinite(*key);
}

// Top-k of one token by warp 0 of the block from the block's shared arrays
// s_ord (order key of every expert, 0 for none; EPL * 32 entries) and s_sc
// (its score): lane l holds the keys of experts l, l + 32, ..., and each of
// the k rounds takes the warp's best (key descending, index ascending),
// removes it at its owner and reads its score, as route_warp_kernel does, so
// the selection, the fp32 slot-order sum and the weights are those bits.
// Lanes j < k write slot j and, when `gmask` is set, token t's bit in the row
// of its expert.  Other warps return at once.
template <int EPL>
__device__ __forceinline__ void warp0_topk_write(const uint32_t* s_ord, const float* s_sc, int t,
                                                 int k, int E, float scale,
                                                 int32_t* __restrict__ idx,
                                                 float* __restrict__ w, uint32_t* gmask) {
  if (threadIdx.x >= 32) return;
  const int lane = threadIdx.x;
  uint32_t ord[EPL];
#pragma unroll
  for (int i = 0; i < EPL; ++i) ord[i] = s_ord[lane + 32 * i];
  int my_e = 0;
  float my_s = 0.f, sum = 0.f;
  for (int j = 0; j < k; ++j) {
    uint32_t bu = 0u;
    int be = INT_MAX;
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
      // increasing i visits increasing experts: ties keep the lower index
      if (ord[i] > bu) {
        bu = ord[i];
        be = lane + 32 * i;
      }
    }
    warp_best(bu, be);
#pragma unroll
    for (int i = 0; i < EPL; ++i)
      if (be == lane + 32 * i) ord[i] = 0u;
    if (!bu) be = INT_MAX;
    const float bs = bu ? s_sc[be] : 0.f;
    if (lane == j) {
      my_e = be;
      my_s = bs;
    }
    sum = (j == 0) ? bs : __fadd_rn(sum, bs);
  }
  if (lane < k) {
    idx[(size_t)t * k + lane] = my_e;
    w[(size_t)t * k + lane] = __fmul_rn(__fdiv_rn(my_s, sum), scale);
    // grouping: token t's bit in the row of each expert it chose
    if (gmask && my_e >= 0 && my_e < E)
      atomicOr(gmask + (size_t)my_e * kPermWords + (t >> 5), 1u << (t & 31));
  }
}

// Routing with one block per token, one thread per expert (EPL * 32 threads,
// EPL = ceil(E / 32)).
//
// With grp.ticket set (T <= kPermBlockTokens), the kernel also groups the
// pairs by expert (group_from_masks) in whichever block finishes last, which
// saves the grouping kernel's launch on small batches.
template <int EPL>
__global__ void __launch_bounds__(1024) route_kernel(
    const float* __restrict__ src, int nsplit, const float* __restrict__ bias, int T, int E,
    int k, float scale, int32_t* __restrict__ idx, float* __restrict__ w,
    int* __restrict__ status, RouteGrouping grp) {
  ptx::pdl_launch_dependents();
  ptx::pdl_wait();
  __shared__ uint32_t s_ord[32 * EPL];
  __shared__ float s_sc[32 * EPL];
  const int t = blockIdx.x;
  const int e = threadIdx.x;
  int bad = 0;
  if (e < E) {
    float key, sc;
    bad = !score_and_key(src, nsplit, (size_t)T * E, (size_t)t * E + e, bias[e], &sc, &key);
    s_ord[e] = key_order(key);
    s_sc[e] = sc;
  } else {
    s_ord[e] = 0u;
  }
  if (__syncthreads_or(bad) && e == 0 && status) atomicOr(status, kStNonFinite);
  warp0_topk_write<EPL>(s_ord, s_sc, t, k, E, scale, idx, w, grp.mask);
  if (!grp.ticket) return;
  // The last block to finish groups every token's pairs by expert.  The
  // block barrier orders this block's index, weight and bit writes before
  // thread 0's ticket, whose release makes them visible GPU-wide; the last
  // block's ticket acquires every other block's writes.
  __shared__ int s_last;
  __syncthreads();
  if (threadIdx.x == 0) s_last = ptx::atom_add_acq_rel_gpu(grp.ticket, 1) == T - 1;
  __syncthreads();
  if (!s_last) return;
  extern __shared__ int grp_smem[];
  group_from_masks(idx, T, E, k, grp.mask, grp.counts, grp.offsets, grp.perm, grp.inv, status,
                   grp.touched, grp_smem);
  if (threadIdx.x == 0) *grp.ticket = 0;  // ready for the next call
}

// Group-limited routing: experts form n_group contiguous groups of E/n_group;
// a group's score is the sum of its two largest keys (its one key for
// one-expert groups); the topk_group groups first under (score descending,
// group index ascending) are kept and the top k is taken among their experts.
__global__ void __launch_bounds__(1024) route_grouped_kernel(
    const float* __restrict__ logits, const float* __restrict__ bias, int T, int E, int k,
    float scale, int n_group, int topk_group, int32_t* __restrict__ idx, float* __restrict__ w,
    int* __restrict__ status) {
  ptx::pdl_launch_dependents();
  ptx::pdl_wait();
  __shared__ uint32_t c_u[kMaxSlots * kMaxSlots];
  __shared__ int c_e[kMaxSlots * kMaxSlots];
  __shared__ float s_sc[1024];
  __shared__ float s_key[1024];
  __shared__ float g_score[32];
  __shared__ int g_keep[32];
  const int t = blockIdx.x;
  const int e = threadIdx.x;
  const int lane = e & 31;
  float key = -INFINITY, sc = 0.f;
  int me = INT_MAX, bad = 0;
  if (e < E) {
    bad = !score_and_key(logits, 1, 0, (size_t)t * E + e, bias[e], &sc, &key);
    me = e;
    s_key[e] = key;
  }
  if (__syncthreads_or(bad) && e == 0 && status) atomicOr(status, kStNonFinite);
  const int G = E / n_group;
  if (e < n_group) {
    float a = -INFINITY, b = -INFINITY;  // two largest keys of group e
    for (int i = e * G; i < (e + 1) * G; ++i) {
      const float v = s_key[i];
      if (v > a) {
        b = a;
        a = v;
      } else if (v > b) {
        b = v;
      }
    }
    g_score[e] = (G == 1) ? a : __fadd_rn(a, b);
    g_keep[e] = 0;
  }
  __syncthreads();
  if (e < 32) {
    bool taken = false;
    for (int j = 0; j < topk_group; ++j) {
      uint32_t bu = (lane < n_group && !taken) ? key_order(g_score[lane]) : 0u;
      int be = (lane < n_group && !taken) ? lane : INT_MAX;
      warp_best(bu, be);
      if (bu && be == lane) taken = true;
    }
    if (lane < n_group) g_keep[lane] = taken ? 1 : 0;
  }
  __syncthreads();
  if (e < E && !g_keep[e / G]) key = -INFINITY;
  block_topk_write(key, sc, me, t, k, scale, idx, w, c_u, c_e, s_sc);
}

// Large batches: one warp per token (four tokens per block), each lane
// holding the experts lane, lane + 32, ...; the same arithmetic in the same
// order as route_kernel, so both give identical bits.
template <int EPL>
__global__ void __launch_bounds__(128) route_warp_kernel(
    const float* __restrict__ src, int nsplit, const float* __restrict__ bias, int T, int E,
    int k, float scale, int32_t* __restrict__ idx, float* __restrict__ w,
    int* __restrict__ status) {
  ptx::pdl_launch_dependents();
  ptx::pdl_wait();
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * 4 + (threadIdx.x >> 5);
  if (t >= T) return;
  const size_t plane = (size_t)T * E;
  float key[EPL], sc[EPL];
  bool bad = false;
#pragma unroll
  for (int i = 0; i < EPL; ++i) {
    const int e = lane + 32 * i;
    if (e < E) {
      const float* p = src + (size_t)t * E + e;
      float l = p[0];
      for (int s0 = 1; s0 < nsplit; s0 += 8) {
        float v[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) v[q] = (s0 + q < nsplit) ? p[(s0 + q) * plane] : 0.f;
#pragma unroll
        for (int q = 0; q < 8; ++q)
          if (s0 + q < nsplit) l = __fadd_rn(l, v[q]);
      }
      const double sd = 1.0 / (1.0 + exp(-(double)l));
      sc[i] = __double2float_rn(sd);
      key[i] = __fadd_rn(sc[i], bias[e]);
      if (!isfinite(l) || !isfinite(key[i])) bad = true;
    } else {
      sc[i] = 0.f;
      key[i] = -INFINITY;
    }
  }
  if (__any_sync(0xffffffffu, bad) && lane == 0 && status) atomicOr(status, kStNonFinite);

  uint32_t ord[EPL];
#pragma unroll
  for (int i = 0; i < EPL; ++i) ord[i] = (lane + 32 * i < E) ? key_order(key[i]) : 0u;
  int my_e = 0;
  float my_s = 0.f, sum = 0.f;
  for (int j = 0; j < k; ++j) {
    uint32_t bu = 0u;
    int be = INT_MAX;
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
      // increasing i visits increasing experts: ties keep the lower index
      if (ord[i] > bu) {
        bu = ord[i];
        be = lane + 32 * i;
      }
    }
    warp_best(bu, be);
    // the owner lane takes the winner out and broadcasts its score
    float os = 0.f;
#pragma unroll
    for (int i = 0; i < EPL; ++i)
      if (be == lane + 32 * i) {
        os = sc[i];
        ord[i] = 0u;
      }
    const float bs = bu ? __shfl_sync(0xffffffffu, os, be & 31) : 0.f;
    if (!bu) be = INT_MAX;
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

template <int EPL>
cudaError_t launch_route_warp(const float* src, int nsplit, const float* bias, int T, int E, int k,
                              float scale, int32_t* idx, float* w, int* status, cudaStream_t st) {
  return launch_pdl(route_warp_kernel<EPL>, dim3((T + 3) / 4), dim3(128), 0, st, src, nsplit, bias,
                    T, E, k, scale, idx, w, status);
}

cudaError_t launch_route_grouped(const float* logits, const float* bias, int T, int E, int k,
                                 float scale, int n_group, int topk_group, int32_t* idx, float* w,
                                 int* status, cudaStream_t st) {
  const int threads = (E + 31) / 32 * 32;
  return launch_pdl(route_grouped_kernel, dim3(T), dim3(threads < 32 ? 32 : threads), 0, st,
                    logits, bias, T, E, k, scale, n_group, topk_group, idx, w, status);
}

// Up to 1024 tokens: a block per token (more threads per token, shorter
// chains); beyond that a warp per token.
constexpr int kRouteBlockPerTokenMaxT = 1024;

// One route_kernel<EPL> launch (EPL = ceil(E / 32) rounded up to a power of
// two, EPL * 32 threads); `grouped`: with the grouping tail and its shared
// memory.
template <int EPL>
cudaError_t launch_route_block(const float* src, int nsplit, const float* bias, int T, int E,
                               int k, float scale, int32_t* idx, float* w, int* status,
                               const RouteGrouping& grp, bool grouped, cudaStream_t st) {
  size_t smem = 0;
  if (grouped) {
    static std::atomic<uint64_t> smem_set{0};
    const cudaError_t e = set_smem_once(route_kernel<EPL>, (int)permute_block_smem(1024), smem_set);
    if (e != cudaSuccess) return e;
    smem = permute_block_smem(E);
  }
  // without the grouping tail only the bitmask rows (if any) are passed on
  RouteGrouping g{};
  if (grouped) g = grp;
  else g.mask = grp.mask;
  return launch_pdl(route_kernel<EPL>, dim3(T), dim3(32 * EPL), smem, st, src, nsplit, bias, T, E,
                    k, scale, idx, w, status, g);
}

cudaError_t launch_route_block_any(const float* src, int nsplit, const float* bias, int T, int E,
                                   int k, float scale, int32_t* idx, float* w, int* status,
                                   const RouteGrouping& grp, bool grouped, cudaStream_t st) {
  const int epl = (E + 31) / 32;
  if (epl <= 1)
    return launch_route_block<1>(src, nsplit, bias, T, E, k, scale, idx, w, status, grp, grouped, st);
  if (epl <= 2)
    return launch_route_block<2>(src, nsplit, bias, T, E, k, scale, idx, w, status, grp, grouped, st);
  if (epl <= 4)
    return launch_route_block<4>(src, nsplit, bias, T, E, k, scale, idx, w, status, grp, grouped, st);
  if (epl <= 8)
    return launch_route_block<8>(src, nsplit, bias, T, E, k, scale, idx, w, status, grp, grouped, st);
  if (epl <= 16)
    return launch_route_block<16>(src, nsplit, bias, T, E, k, scale, idx, w, status, grp, grouped, st);
  return launch_route_block<32>(src, nsplit, bias, T, E, k, scale, idx, w, status, grp, grouped, st);
}

cudaError_t launch_route(const float* src, int nsplit, const float* bias, int T, int E, int k,
                         float scale, int32_t* idx, float* w, int* status, cudaStream_t st) {
  if (T <= kRouteBlockPerTokenMaxT)
    return launch_route_block_any(src, nsplit, bias, T, E, k, scale, idx, w, status,
                                  RouteGrouping{}, false, st);
  const int epl = (E + 31) / 32;
  if (epl <= 1) return launch_route_warp<1>(src, nsplit, bias, T, E, k, scale, idx, w, status, st);
  if (epl <= 2) return launch_route_warp<2>(src, nsplit, bias, T, E, k, scale, idx, w, status, st);
  if (epl <= 4) return launch_route_warp<4>(src, nsplit, bias, T, E, k, scale, idx, w, status, st);
  if (epl <= 8) return launch_route_warp<8>(src, nsplit, bias, T, E, k, scale, idx, w, status, st);
  if (epl <= 16) return launch_route_warp<16>(src, nsplit, bias, T, E, k, scale, idx, w, status, st);
  return launch_route_warp<32>(src, nsplit, bias, T, E, k, scale, idx, w, status, st);
}

cudaError_t launch_route_bits(const float* src, int nsplit, const float* bias, int T, int E,
                              int k, float scale, int32_t* idx, float* w, int* status,
                              uint32_t* mask, cudaStream_t st) {
  if (T > kPermBlockTokens || !mask) return cudaErrorInvalidValue;
  RouteGrouping grp{};
  grp.mask = mask;
  return launch_route_block_any(src, nsplit, bias, T, E, k, scale, idx, w, status, grp, false, st);
}

cudaError_t launch_route_and_group(const float* src, int nsplit, const float* bias, int T, int E,
                                   int k, float scale, int32_t* idx, float* w, int* status,
                                   const RouteGrouping& grp, cudaStream_t st) {
  if (T > kPermBlockTokens || !grp.ticket || !grp.mask) return cudaErrorInvalidValue;
  return launch_route_block_any(src, nsplit, bias, T, E, k, scale, idx, w, status, grp, true, st);
}

}  // namespace moe
