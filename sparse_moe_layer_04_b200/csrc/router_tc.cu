// Router logits for small batches in one tensor-core kernel that reads the
// fp32 router weight itself.
//
//   logits[t, e] = sum_d h[t, d] * Wr[e, d]      ("Routing: learned", MoE
//   panel of "Model anatomy -- GLM-5.2"; the router stays fp32)
//
// h is bf16, so every product is exact once Wr is written as three bf16
// pieces, w = hi + mid + lo (hi = bf16(w), mid = bf16(w - hi), lo =
// bf16(w - hi - mid); both subtractions are exact and |w - (hi+mid+lo)| <=
// 2^-24 |w|).  The kernel splits each K-block of Wr in shared memory as it
// arrives, so no split copy of the weight is written or read back.  The
// three piece tiles of a K-block lie one after the other and form a single
// 192-row B operand: one tcgen05.mma (M = 128, N = 192, K = 16) per K-step
// accumulates h . hi, h . mid and h . lo into three 64-column fp32
// accumulators, which the epilogue adds as (hi + mid) + lo.
//
// Grid: (E / 64 expert columns) x (nsplit K ranges) x (row tiles of 128
// tokens).  A CTA owns one 128 x 64 output tile over kb_per K-blocks of 64
// and writes it to its own partial-sum plane [nsplit][T][E]; the routing
// kernel adds the planes in plane order.  Every K-block of the CTA has its
// own buffers (at most kMaxKb of them), so each barrier completes exactly
// once and no buffer is reused.
//
// Roles (256 threads):
//   warp 0 lane 0   TMA: the h tile (128 x 64 bf16) and the Wr tile (64 x 64
//                   fp32, two 64 x 32 boxes) of every K-block, all at once.
//   warp 1          TMEM allocation (256 columns); lane 0 issues the 4
//                   K-steps of each K-block.
//   warps 4-7       split: thread i takes 32 weights (one box row) of row
//                   i / 2 of each K-block and writes their three pieces into
//                   the piece tiles (128-byte swizzled bf16); then the
//                   epilogue (warp w reads TMEM lanes 32 (w % 4) ..) stores the
//                   plane rows.
#include <cuda_bf16.h>

#include "ffn_common.cuh"
#include "moe_internal.cuh"
#include "sm100_ptx.cuh"

namespace moe {
namespace {

constexpr int kRtN = 64;                    // experts per CTA
constexpr int kRtM = 128;                   // tokens per CTA
constexpr int kRtBK = 64;                   // K-block
constexpr int kMaxKb = 4;                   // K-blocks per CTA (buffers)
constexpr int kRtThreads = 256;
constexpr int kASz = kRtM * kRtBK * 2;      // 16 KB h tile
constexpr int kWSz = kRtN * kRtBK * 4;      // 16 KB fp32 weight tile (two 8 KB boxes)
constexpr int kPSz = kRtN * kRtBK * 2;      // 8 KB bf16 piece tile
constexpr uint32_t kRtIdesc = ptx::idesc_bf16_f32(kRtM, 3 * kRtN);
constexpr uint32_t kRtTmemCols = 256;       // three 64-column accumulators

struct RouterTcParams {
  CUtensorMap a;      // h [T, D] bf16, box 64 x 128, 128-byte swizzle
  CUtensorMap w;      // Wr [E, D] fp32, box 32 x 64, 128-byte swizzle
  float* partials;    // [nsplit][T][E]
  int* status;        // nullable
  int T, E, kb_total, kb_per;
};

struct RouterTcShared {
  uint64_t full[kMaxKb];    // h and Wr tiles of K-block kb landed
  uint64_t split[kMaxKb];   // its three pieces are written (128 arrivals)
  uint64_t acc;             // every MMA of the CTA has completed
  uint32_t tmem_base;
  int abort;
};

constexpr size_t kRtSmem = 1024 + (size_t)kMaxKb * (kASz + kWSz + 3 * kPSz) + sizeof(RouterTcShared);
static_assert(kRtSmem <= 227 * 1024, "shared memory budget");

__device__ __forceinline__ uint32_t bf16x2_bits(__nv_bfloat162 v) {
  return *reinterpret_cast<uint32_t*>(&v);
}

__global__ void __launch_bounds__(kRtThreads, 1)
    router_tc_kernel(const __grid_constant__ RouterTcParams p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = ptx::smem_addr(smem_raw);
  uint8_t* base = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
  uint8_t* s_a = base;                                  // [kMaxKb][kASz]
  uint8_t* s_w = s_a + kMaxKb * kASz;                   // [kMaxKb][kWSz]
  uint8_t* s_p = s_w + kMaxKb * kWSz;                   // [kMaxKb][3][kPSz]
  RouterTcShared& ss = *reinterpret_cast<RouterTcShared*>(s_p + kMaxKb * 3 * kPSz);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n0 = blockIdx.x * kRtN, split = blockIdx.y, m0 = blockIdx.z * kRtM;
  const int kb0 = split * p.kb_per;
  const int nkb = min(p.kb_per, p.kb_total - kb0);

  ptx::pdl_launch_dependents();
  if (warp == 1) {
    ptx::tmem_alloc(&ss.tmem_base, kRtTmemCols);
    ptx::tmem_relinquish();
  }
  if (threadIdx.x == 0) {
    for (int i = 0; i < kMaxKb; ++i) {
      ptx::mbar_init(&ss.full[i], 1);
      ptx::mbar_init(&ss.split[i], 128);
    }
    ptx::mbar_init(&ss.acc, 1);
    ss.abort = 0;
    ptx::fence_barrier_init();
  }
  if (threadIdx.x == 32) {
    ptx::tma_prefetch_desc(&p.a);
    ptx::tma_prefetch_desc(&p.w);
  }
  ptx::pdl_wait();
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = ss.tmem_base;
  volatile int* abort = &ss.abort;

  if (warp == 0) {
    if (lane == 0) {
      for (int kb = 0; kb < nkb; ++kb) {
        const int x = (kb0 + kb) * kRtBK;
        ptx::mbar_arrive_expect_tx(&ss.full[kb], kASz + kWSz);
        ptx::tma_load_2d(s_a + kb * kASz, &p.a, &ss.full[kb], x, m0);
        ptx::tma_load_2d(s_w + kb * kWSz, &p.w, &ss.full[kb], x, n0);
        ptx::tma_load_2d(s_w + kb * kWSz + kWSz / 2, &p.w, &ss.full[kb], x + 32, n0);
      }
      // every load has landed before the CTA may retire
      for (int kb = 0; kb < nkb; ++kb) ffn::wait_drain(&ss.full[kb], 0, abort);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      uint32_t accumulate = 0;
      for (int kb = 0; kb < nkb; ++kb) {
        if (!ptx::mbar_wait(&ss.full[kb], 0, abort) || !ptx::mbar_wait(&ss.split[kb], 0, abort))
          break;
        ptx::tc_fence_after();
        const uint64_t a_desc = ptx::smem_desc_sw128(ptx::smem_addr(s_a + kb * kASz));
        const uint64_t p_desc = ptx::smem_desc_sw128(ptx::smem_addr(s_p + kb * 3 * kPSz));
#pragma unroll
        for (int kk = 0; kk < kRtBK / 16; ++kk) {
          ptx::mma_f16_ss(tmem, a_desc + 2 * kk, p_desc + 2 * kk, kRtIdesc, accumulate);
          accumulate = 1;
        }
      }
      ptx::mma_commit(&ss.acc);
      ffn::wait_drain(&ss.acc, 0, abort);   // no MMA in flight when TMEM is freed
    }
  } else if (warp >= 4) {
    // ---- split of the weight tiles ----
    const int c = threadIdx.x - 128;
    const int r = c >> 1, q = c & 1;        // weight row, 32-wide K half (fp32 box q)
    const uint32_t sw = r & 7;
    bool ok = true;
    for (int kb = 0; kb < nkb; ++kb) {
      if (!ptx::mbar_wait(&ss.full[kb], 0, abort)) {
        ok = false;
        break;
      }
      // row r of fp32 box q: chunk j (4 weights) sits at j ^ (row & 7)
      const uint8_t* wrow = s_w + kb * kWSz + q * (kWSz / 2) + r * 128;
      uint8_t* prow = s_p + kb * 3 * kPSz + r * 128;
#pragma unroll
      for (int j2 = 0; j2 < 4; ++j2) {
        // fp32 chunks 2 j2, 2 j2 + 1 -> bf16 chunk 4 q + j2 of each piece
        const float4 f0 = *reinterpret_cast<const float4*>(wrow + (((2 * j2) ^ sw) << 4));
        const float4 f1 = *reinterpret_cast<const float4*>(wrow + (((2 * j2 + 1) ^ sw) << 4));
        const float v[8] = {f0.x, f0.y, f0.z, f0.w, f1.x, f1.y, f1.z, f1.w};
        // two weights per conversion instruction (bf16x2, round to nearest
        // even); the bf16 -> fp32 widening is exact
        uint32_t pk[3][4];
#pragma unroll
        for (int i = 0; i < 8; i += 2) {
          const float2 x = make_float2(v[i], v[i + 1]);
          const __nv_bfloat162 bh = __float22bfloat162_rn(x);
          const float2 fh = __bfloat1622float2(bh);
          const float2 r1 = make_float2(__fsub_rn(x.x, fh.x), __fsub_rn(x.y, fh.y));
          const __nv_bfloat162 bm = __float22bfloat162_rn(r1);
          const float2 fm = __bfloat1622float2(bm);
          const float2 r2 = make_float2(__fsub_rn(r1.x, fm.x), __fsub_rn(r1.y, fm.y));
          const __nv_bfloat162 bl = __float22bfloat162_rn(r2);
          pk[0][i / 2] = bf16x2_bits(bh);
          pk[1][i / 2] = bf16x2_bits(bm);
          pk[2][i / 2] = bf16x2_bits(bl);
        }
        const uint32_t off = ((4 * q + j2) ^ sw) << 4;
#pragma unroll
        for (int piece = 0; piece < 3; ++piece)
          *reinterpret_cast<uint4*>(prow + piece * kPSz + off) =
              make_uint4(pk[piece][0], pk[piece][1], pk[piece][2], pk[piece][3]);
      }
      ptx::fence_proxy_async_shared();   // the tensor core reads what was written
      ptx::mbar_arrive(&ss.split[kb]);
    }
    // ---- epilogue: row t of the tile, 64 experts, (hi + mid) + lo ----
    // (the warp agrees first: tcgen05.ld is executed by all its lanes or none)
    const bool got = __all_sync(0xffffffffu, ok && ptx::mbar_wait(&ss.acc, 0, abort));
    if (got) {
      ptx::tc_fence_after();
      const int quarter = warp & 3;
      const uint32_t taddr = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
      const int t = m0 + quarter * 32 + lane;
      const bool store = t < p.T && !*abort;
      float4* dst = reinterpret_cast<float4*>(p.partials + ((size_t)split * p.T + t) * p.E + n0);
#pragma unroll 1
      for (int j0 = 0; j0 < kRtN; j0 += 16) {
        uint32_t vh[16], vm[16], vl[16];
        ptx::tmem_ld_x16(taddr + j0, vh);
        ptx::tmem_ld_x16(taddr + kRtN + j0, vm);
        ptx::tmem_ld_x16(taddr + 2 * kRtN + j0, vl);
        ptx::tmem_wait_ld();
        float o[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          o[i] = __fadd_rn(__fadd_rn(__uint_as_float(vh[i]), __uint_as_float(vm[i])),
                           __uint_as_float(vl[i]));
        if (store) {
#pragma unroll
          for (int i = 0; i < 4; ++i)
            dst[j0 / 4 + i] = make_float4(o[4 * i], o[4 * i + 1], o[4 * i + 2], o[4 * i + 3]);
        }
      }
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, kRtTmemCols);
  }
  if (threadIdx.x == 0 && ss.abort && p.status) atomicOr(p.status, kStTimeout);
}

}  // namespace

bool router_tc_shape_ok(int T, int D, int E) {
  return T >= 1 && T <= kRouterTcMaxT && D % kRtBK == 0 && E % kRtN == 0;
}

// K-blocks per plane: one wave of CTAs on the SMs the shared experts' FFN
// leaves free when it runs beside the routing, at most kMaxKb K-blocks each.
void router_tc_split(int T, int D, int E, int* nsplit, int* kb_per) {
  const int kb_total = D / kRtBK;
  const int tiles = (E / kRtN) * ((T + kRtM - 1) / kRtM);
  int want = (kSplitTargetBlocks - kSharedCtas) / (tiles > 0 ? tiles : 1);
  if (want < 1) want = 1;
  int per = (kb_total + want - 1) / want;
  if (per > kMaxKb) per = kMaxKb;
  if (per < 1) per = 1;
  *kb_per = per;
  *nsplit = (kb_total + per - 1) / per;
}

cudaError_t launch_router_tc_fused(const uint16_t* h, const float* Wr, int T, int D, int E,
                                   int nsplit, int kb_per, float* partials, int* status,
                                   cudaStream_t st, const char** why) {
  RouterTcParams p{};
  if (!make_tensor_map(&p.a, h, T, D, kRtM, kRtBK, 2, 128) ||
      !make_tensor_map(&p.w, Wr, E, D, kRtN, 32, 4, 128)) {
    *why = "cuTensorMapEncodeTiled failed for a router operand";
    return cudaErrorInvalidValue;
  }
  p.partials = partials;
  p.status = status;
  p.T = T;
  p.E = E;
  p.kb_total = D / kRtBK;
  p.kb_per = kb_per;
  static std::atomic<uint64_t> smem_set{0};
  const cudaError_t e = set_smem_once(router_tc_kernel, (int)kRtSmem, smem_set);
  if (e != cudaSuccess) return e;
  const dim3 grid(E / kRtN, nsplit, (T + kRtM - 1) / kRtM);
  return launch_pdl(router_tc_kernel, grid, dim3(kRtThreads), kRtSmem, st, p);
}

}  // namespace moe
