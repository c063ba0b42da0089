// Grouped expert GEMMs on the 5th-generation tensor cores (tcgen05 + TMEM),
// operands staged by TMA.
//
// The expert MLP is y = w2 (silu(w1 x) * (w3 x)) with w1/w3 the input
// projections and w2 the output projection ("GLM-5.2", PocketLLM,
// Implemented execution path, names w1/w3 and w2; the gated form is the
// reading taken where the pages are silent).  The routed experts see only the
// rows grouped to them; the always-on shared expert sees every token ("Model
// anatomy -- GLM-5.2", MoE panel, and "Expert fan-out 8 + 1").
//
// One persistent kernel runs up to two grouped GEMM "problems" back to back
// in a single tile space:
//   problem 0 (gate/up): act[r, n] = silu(A[r] . W1[e][n]) * (A[r] . W3[e][n])
//             128 x N/2 output tile; the W1 and W3 row blocks of the tile are
//             stacked into one N-row B operand, so one MMA feeds both
//             accumulators (TMEM columns [0, N/2) gate, [N/2, N) up) and the
//             epilogue applies the SiLU gate and rounds to bf16.
//   problem 1 (down):    y[r, n] = act[r] . W2[e][n], 128 x N fp32 tile.
// Tiles are numbered problem 0 first, then problem 1; within a problem routed
// experts first (expert, column tile, row tile with the row tile fastest, so
// CTAs running at the same time share each weight tile through L2), then the
// shared experts.  CTA c takes tiles c, c + gridDim.x, ...  A down tile of an
// expert waits until every gate/up tile of that expert has been stored: each
// gate/up epilogue warp releases a per-expert counter after a proxy fence, and
// the producer acquires it before its TMA loads read the activations.  Down tiles
// therefore fill the SMs that the tail of the gate/up tiles leaves idle.
// Because every CTA takes its tiles in increasing order and all CTAs are
// resident (one per SM), every counter a CTA waits on is advanced by tiles that
// precede it, so the waits always end; they are bounded all the same.
//
// N (the MMA width) is 256 for large batches and 128 for small ones, where
// each expert has only a row tile or two and the weight stream must be cut
// finer to keep all 148 SMs busy.  The same kernel also computes the router
// logits as a dense split-K GEMM (one problem, one shared group per K chunk).
//
// CTA structure (192 threads, one CTA per SM):
//   warp 0      TMA producer: ring of (A 128x64, B Nx64) bf16 tiles (4 stages
//               for N = 256, 6 for N = 128), 128-byte swizzled, completion
//               counted on "full" mbarriers.
//   warp 1      TMEM allocator and single-thread MMA issuer:
//               tcgen05.mma.cta_group::1.kind::f16, M = 128, N, K = 16,
//               fp32 accumulators in TMEM, two accumulator buffers so the
//               epilogue of tile i overlaps the main loop of tile i+1.
//   warps 2-5   epilogue: tcgen05.ld of the accumulator (warp w reads TMEM
//               lanes 32*(w%4) .. +31), fused activation, global stores.
#include <cuda_bf16.h>

#include "moe_internal.cuh"
#include "sm100_ptx.cuh"

namespace moe {
namespace {

constexpr int BM = 128;
constexpr int BK = 64;                    // one 128-byte swizzle row of bf16
constexpr int THREADS = 192;
constexpr int A_BYTES = BM * BK * 2;      // 16 KiB
constexpr int MAX_E = 1024;
constexpr int RING_BYTES = 192 * 1024;    // operand ring budget
constexpr int MAX_STAGES = 6;
constexpr int EPI_WARPS = 4;              // each releases its rows of a gate/up tile

template <int MMA_N>
struct Shape {
  static constexpr int B_BYTES = MMA_N * BK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int STAGES = RING_BYTES / STAGE_BYTES;    // 4 (N=256) or 6 (N=128)
  static constexpr int ACC_COLS = MMA_N;                     // fp32 TMEM columns per accumulator
  static constexpr uint32_t TMEM_COLS = 2 * ACC_COLS;        // double buffered
  static constexpr uint32_t IDESC = ptx::idesc_bf16_f32(BM, MMA_N);
};

// One grouped GEMM.  Routed group e has rows [off[e], off[e+1]) of the routed
// A / output matrices; shared group s has rows s*T .. s*T + T - 1 of the
// shared output (its A rows start at s * a_s_group_stride).
struct alignas(64) Problem {
  CUtensorMap a_r;   // routed A  [rows_r, K_r]
  CUtensorMap a_s;   // shared A
  CUtensorMap b0_r;  // W1 [E*F, D] (gate/up) | W2 [E*D, F] (down)
  CUtensorMap b1_r;  // W3 [E*F, D] (gate/up only)
  CUtensorMap b0_s;  // Ws1 | Ws2
  CUtensorMap b1_s;  // Ws3
  void* out_r;
  void* out_s;
  int K_r, K_s;              // reduction lengths
  int N_r, N_s;              // output columns (= output row strides)
  int a_s_group_stride;      // rows between shared groups' A blocks (0 or T)
  int b_r_group_rows;        // B rows per routed expert (F or D)
  int b_s_group_rows;        // B rows per shared expert (Fs, D or 0)
  int bn_out;                // output columns per tile (N or N/2)
  int k_chunk;               // > 0: shared group g covers K range [g*k_chunk, (g+1)*k_chunk)
  int a_k_mod;               // > 0: the A operand's K coordinate wraps modulo this
  int gateup;                // epilogue: 1 = SiLU gate -> bf16, 0 = fp32 store
};

struct GemmParams {
  Problem pr[2];
  const int32_t* offsets;    // [E+1] routed group row offsets (E > 0)
  int* status;
  int* counters;             // [E+S] gate/up tiles stored per group (two problems)
  int nprob;                 // 1 or 2
  int E, S, T;
  int rows_r;                // T * k
};

struct SharedState {
  uint64_t full[MAX_STAGES];
  uint64_t empty[MAX_STAGES];
  uint64_t tmem_full[2];
  uint64_t tmem_empty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
  int mt_total;              // routed row tiles over all experts
  int off[MAX_E + 1];        // group row offsets
  int mt_prefix[MAX_E + 1];  // routed row-tile prefix per expert
};

struct TileInfo {
  int prob;
  bool shared;
  int grp;      // expert (routed) or shared expert index
  int m0;       // first row within the group
  int n0;       // first output column
  int rows;     // rows in the group
  int row0;     // group's first row in the output (and routed A) matrix
  int mt;       // row tiles of the group
};

__device__ __forceinline__ int col_tiles(int N, int bn) { return (N + bn - 1) / bn; }

__device__ __forceinline__ int problem_tiles(const Problem& P, const SharedState& ss,
                                             const GemmParams& p) {
  const int mt_s = (p.T + BM - 1) / BM;
  return ss.mt_total * col_tiles(P.N_r, P.bn_out) + p.S * mt_s * col_tiles(P.N_s, P.bn_out);
}

__device__ __forceinline__ TileInfo decode_tile(int tile, const SharedState& ss,
                                                const GemmParams& p, int tiles0) {
  TileInfo ti;
  ti.prob = (tile >= tiles0) ? 1 : 0;
  const Problem& P = p.pr[ti.prob];
  const int lt = tile - (ti.prob ? tiles0 : 0);
  const int nt_r = col_tiles(P.N_r, P.bn_out);
  const int routed = ss.mt_total * nt_r;
  if (lt < routed) {
    // expert e: largest with mt_prefix[e] * nt_r <= lt
    const int q = lt / nt_r;
    int lo = 0, hi = p.E - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (ss.mt_prefix[mid] <= q) lo = mid; else hi = mid - 1;
    }
    const int e = lo;
    const int rows = ss.off[e + 1] - ss.off[e];
    const int mt = (rows + BM - 1) / BM;
    const int local = lt - ss.mt_prefix[e] * nt_r;
    ti.shared = false;
    ti.grp = e;
    ti.m0 = (local % mt) * BM;
    ti.n0 = (local / mt) * P.bn_out;
    ti.rows = rows;
    ti.row0 = ss.off[e];
    ti.mt = mt;
  } else {
    const int ls = lt - routed;
    const int mt = (p.T + BM - 1) / BM;
    const int nt = col_tiles(P.N_s, P.bn_out);
    const int s = ls / (mt * nt);
    const int rem = ls - s * mt * nt;
    ti.shared = true;
    ti.grp = s;
    ti.m0 = (rem % mt) * BM;
    ti.n0 = (rem / mt) * P.bn_out;
    ti.rows = p.T;
    ti.row0 = s * p.T;
    ti.mt = mt;
  }
  return ti;
}

// K range of a tile: the whole reduction, or one chunk of it when the shared
// groups split K (the router's split-K partial sums).
__device__ __forceinline__ void tile_k_range(const TileInfo& ti, const Problem& P, int* kbeg,
                                             int* K) {
  if (ti.shared && P.k_chunk > 0) {
    *kbeg = ti.grp * P.k_chunk;
    *K = min(P.k_chunk, P.K_s - *kbeg);
  } else {
    *kbeg = 0;
    *K = ti.shared ? P.K_s : P.K_r;
  }
}

__device__ __forceinline__ float silu_times(float g, float u) {
  return g / (1.0f + __expf(-g)) * u;
}

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&v);
}

// Waits for in-flight async work even after an abort (bounded by the same
// clock budget); a timeout here raises the CTA's abort flag too.
__device__ __forceinline__ void wait_drain(uint64_t* bar, uint32_t parity, volatile int* abort) {
  int ignore_abort = 0;
  if (!ptx::mbar_wait(bar, parity, &ignore_abort)) *abort = 1;
}

template <int MMA_N>
__global__ void __launch_bounds__(THREADS, 1) grouped_gemm_kernel(const __grid_constant__ GemmParams p) {
  using Sh = Shape<MMA_N>;
  constexpr int STAGES = Sh::STAGES;
  constexpr int STAGE_BYTES = Sh::STAGE_BYTES;
  constexpr int ACC_COLS = Sh::ACC_COLS;
  constexpr uint32_t TMEM_COLS = Sh::TMEM_COLS;
  constexpr uint32_t IDESC = Sh::IDESC;
  constexpr int HALF = MMA_N / 2;  // gate/up: W1 rows [0, HALF), W3 rows [HALF, MMA_N)
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte aligned operand ring (128-byte swizzle atoms span 1024 bytes)
  const uint32_t raw_addr = ptx::smem_addr(smem_raw);
  uint8_t* ring = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
  SharedState& ss = *reinterpret_cast<SharedState*>(ring + STAGES * STAGE_BYTES);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  ptx::pdl_launch_dependents();
  if (warp == 1) {
    ptx::tmem_alloc(&ss.tmem_base, TMEM_COLS);
    ptx::tmem_relinquish();
  }
  if (threadIdx.x == 0) {
    for (int i = 0; i < STAGES; ++i) {
      ptx::mbar_init(&ss.full[i], 1);
      ptx::mbar_init(&ss.empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(&ss.tmem_full[i], 1);
      ptx::mbar_init(&ss.tmem_empty[i], 4);
    }
    ptx::mbar_init(&ss.drain, 1);
    ss.abort = 0;
    ptx::fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    ptx::tma_prefetch_desc(&p.pr[0].a_r);
    ptx::tma_prefetch_desc(&p.pr[0].b0_r);
    ptx::tma_prefetch_desc(&p.pr[0].b1_r);
  }
  // everything below reads what earlier kernels in the stream wrote
  ptx::pdl_wait();

  // Routed row-tile prefix from the group offsets (warp 2 scans 32 experts at a time).
  if (warp == 2) {
    int carry = 0;
    bool bad = false;
    for (int base = 0; base < p.E; base += 32) {
      const int e = base + lane;
      int cnt = 0;
      if (e < p.E) {
        const int a = p.offsets[e], b = p.offsets[e + 1];
        ss.off[e] = a;
        if (e == p.E - 1) ss.off[p.E] = b;
        if (a < 0 || b < a || b > p.rows_r || (e == 0 && a != 0)) bad = true;
        cnt = b >= a ? (b - a + BM - 1) / BM : 0;
      }
      int incl = cnt;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += v;
      }
      if (e < p.E) ss.mt_prefix[e] = carry + incl - cnt;
      carry += __shfl_sync(0xffffffffu, incl, 31);
    }
    bad = __any_sync(0xffffffffu, bad);
    if (lane == 0) {
      ss.mt_prefix[p.E] = carry;
      ss.mt_total = bad ? 0 : carry;
      if (bad && p.status) atomicOr(p.status, kStBounds);
    }
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();

  const uint32_t tmem_base = ss.tmem_base;
  const int tiles0 = problem_tiles(p.pr[0], ss, p);
  const int total = tiles0 + (p.nprob > 1 ? problem_tiles(p.pr[1], ss, p) : 0);
  volatile int* abort = &ss.abort;

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued_mask = 0, last_parity = 0;
      for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
        const TileInfo ti = decode_tile(tile, ss, p, tiles0);
        const Problem& P = p.pr[ti.prob];
        if (ti.prob == 1) {
          // the activations of this group come from problem 0's epilogues
          const int g = ti.shared ? p.E + ti.grp : ti.grp;
          const int nt0 = ti.shared ? col_tiles(p.pr[0].N_s, p.pr[0].bn_out)
                                    : col_tiles(p.pr[0].N_r, p.pr[0].bn_out);
          if (!ptx::counter_wait(p.counters + g, EPI_WARPS * ti.mt * nt0, abort)) break;
          ptx::fence_proxy_async_global();
        }
        const CUtensorMap* amap = ti.shared ? &P.a_s : &P.a_r;
        const CUtensorMap* b0 = ti.shared ? &P.b0_s : &P.b0_r;
        const CUtensorMap* b1 = ti.shared ? &P.b1_s : &P.b1_r;
        const int a_row = ti.shared ? ti.grp * P.a_s_group_stride + ti.m0 : ti.row0 + ti.m0;
        const int b_row = ti.grp * (ti.shared ? P.b_s_group_rows : P.b_r_group_rows) + ti.n0;
        int kbeg, K;
        tile_k_range(ti, P, &kbeg, &K);
        const int nk = (K + BK - 1) / BK;
        bool ok = true;
        for (int kb = 0; kb < nk; ++kb) {
          if (!ptx::mbar_wait(&ss.empty[stage], phase ^ 1u, abort)) { ok = false; break; }
          uint8_t* sa = ring + stage * STAGE_BYTES;
          uint8_t* sb = sa + A_BYTES;
          const int xb = kbeg + kb * BK;
          const int xa = P.a_k_mod > 0 ? xb % P.a_k_mod : xb;
          ptx::mbar_arrive_expect_tx(&ss.full[stage], STAGE_BYTES);
          ptx::tma_load_2d(sa, amap, &ss.full[stage], xa, a_row);
          if (P.gateup) {
            ptx::tma_load_2d(sb, b0, &ss.full[stage], xb, b_row);
            ptx::tma_load_2d(sb + HALF * BK * 2, b1, &ss.full[stage], xb, b_row);
          } else {
            ptx::tma_load_2d(sb, b0, &ss.full[stage], xb, b_row);
          }
          issued_mask |= 1u << stage;
          last_parity = (last_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
      }
      // every issued load has landed before the CTA may retire
      for (int s = 0; s < STAGES; ++s)
        if (issued_mask & (1u << s)) wait_drain(&ss.full[s], (last_parity >> s) & 1u, abort);
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
        const TileInfo ti = decode_tile(tile, ss, p, tiles0);
        int kbeg, K;
        tile_k_range(ti, p.pr[ti.prob], &kbeg, &K);
        const int nk = (K + BK - 1) / BK;
        if (!ptx::mbar_wait(&ss.tmem_empty[acc], acc_phase ^ 1u, abort)) break;
        ptx::tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * ACC_COLS;
        bool ok = true;
        for (int kb = 0; kb < nk; ++kb) {
          if (!ptx::mbar_wait(&ss.full[stage], phase, abort)) { ok = false; break; }
          ptx::tc_fence_after();
          const uint32_t sa = ptx::smem_addr(ring + stage * STAGE_BYTES);
          const uint32_t sb = sa + A_BYTES;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            ptx::mma_f16_ss(d_tmem, ptx::smem_desc_sw128(sa + kk * 32),
                            ptx::smem_desc_sw128(sb + kk * 32), IDESC,
                            (kb > 0 || kk > 0) ? 1u : 0u);
          }
          ptx::mma_commit(&ss.empty[stage]);   // frees the smem stage when these MMAs finish
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        ptx::mma_commit(&ss.tmem_full[acc]);   // accumulator ready for the epilogue
        if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
      }
      ptx::mma_commit(&ss.drain);
      wait_drain(&ss.drain, 0, abort);
    }
  } else {
    // ---------------- epilogue (warps 2..5) ----------------
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
      const TileInfo ti = decode_tile(tile, ss, p, tiles0);
      const Problem& P = p.pr[ti.prob];
      if (!ptx::mbar_wait(&ss.tmem_full[acc], acc_phase, abort)) break;
      ptx::tc_fence_after();
      const int r = ti.m0 + q * 32 + lane;       // row within the group
      const bool row_ok = r < ti.rows;
      const int N = ti.shared ? P.N_s : P.N_r;
      const size_t out_row = (size_t)ti.row0 + r;
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + acc * ACC_COLS;
      if (P.gateup) {
        uint16_t* out = static_cast<uint16_t*>(ti.shared ? P.out_s : P.out_r);
#pragma unroll 1
        for (int c = 0; c < HALF; c += 16) {
          uint32_t g[16], u[16];
          ptx::tmem_ld_x16(taddr + c, g);
          ptx::tmem_ld_x16(taddr + HALF + c, u);
          ptx::tmem_wait_ld();
          const int col = ti.n0 + c;
          if (row_ok && col < N) {
            uint32_t pk[8];
#pragma unroll
            for (int i = 0; i < 8; ++i)
              pk[i] = pack_bf16(silu_times(__uint_as_float(g[2 * i]), __uint_as_float(u[2 * i])),
                                silu_times(__uint_as_float(g[2 * i + 1]),
                                           __uint_as_float(u[2 * i + 1])));
            uint4* dst = reinterpret_cast<uint4*>(out + out_row * N + col);
            dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
            if (col + 8 < N) dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
          }
        }
      } else {
        float* out = static_cast<float*>(ti.shared ? P.out_s : P.out_r);
#pragma unroll 1
        for (int c = 0; c < MMA_N; c += 16) {
          uint32_t v[16];
          ptx::tmem_ld_x16(taddr + c, v);
          ptx::tmem_wait_ld();
          const int col = ti.n0 + c;
          if (row_ok && col < N) {
            uint4* dst = reinterpret_cast<uint4*>(out + out_row * N + col);
            dst[0] = make_uint4(v[0], v[1], v[2], v[3]);
            dst[1] = make_uint4(v[4], v[5], v[6], v[7]);
            if (col + 8 < N) {
              dst[2] = make_uint4(v[8], v[9], v[10], v[11]);
              dst[3] = make_uint4(v[12], v[13], v[14], v[15]);
            }
          }
        }
      }
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&ss.tmem_empty[acc]);
      if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
      if (p.nprob > 1 && ti.prob == 0) {
        // release this warp's rows of the tile to the down tiles of its
        // group: make the stores visible to the async proxy and to the whole
        // GPU, then count them (four counts per tile, one per epilogue warp)
        ptx::fence_proxy_async_global();
        __threadfence();
        __syncwarp();
        if (lane == 0) atomicAdd(p.counters + (ti.shared ? p.E + ti.grp : ti.grp), 1);
      }
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem_base, TMEM_COLS);
  }
  if (threadIdx.x == 0 && ss.abort && p.status) atomicOr(p.status, kStTimeout);
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  return fn;
}

// bf16 row-major [rows, cols] matrix, box = box_rows x 64 columns, 128-byte swizzle.
bool make_map(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * 2};
  const cuuint32_t box[2] = {BK, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int MMA_N>
constexpr size_t smem_bytes() {
  return 1024 + Shape<MMA_N>::STAGES * Shape<MMA_N>::STAGE_BYTES + sizeof(SharedState);
}
static_assert(smem_bytes<256>() <= 227 * 1024 && smem_bytes<128>() <= 227 * 1024,
              "shared memory budget");

template <int MMA_N>
cudaError_t launch_one(const GemmParams& p, int tiles_upper, cudaStream_t st) {
  static int configured_dev = -1;
  int dev = 0;
  cudaGetDevice(&dev);
  if (configured_dev != dev) {
    cudaError_t e = cudaFuncSetAttribute(grouped_gemm_kernel<MMA_N>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem_bytes<MMA_N>());
    if (e != cudaSuccess) return e;
    configured_dev = dev;
  }
  int grid = num_sms();
  if (tiles_upper < grid) grid = tiles_upper;
  if (grid < 1) grid = 1;
  return launch_pdl(grouped_gemm_kernel<MMA_N>, dim3(grid), dim3(THREADS), smem_bytes<MMA_N>(),
                    st, p);
}

}  // namespace

// Router logits on the tensor cores.  The fp32 router weight is split exactly
// into three bf16 pieces (hi + mid + lo, each the bf16 rounding of what the
// previous pieces leave; together they carry the 24-bit fp32 significand),
// stored side by side as wr3 [E, 3D].  h is bf16 and so exact in the MMA, so
//   logits = [h | h | h] . wr3^T
// is a dense GEMM over K' = 3D with fp32 accumulation.  It runs as `nsplit`
// shared groups that each take one K' chunk and write their own partial-sum
// plane [T, E]; the consumer adds the planes in order.
cudaError_t launch_router_tc(const uint16_t* h, const uint16_t* wr3, int T, int D, int E,
                             int nsplit, int chunk, float* partials, cudaStream_t st,
                             const char** why) {
  const int bn = router_tile_n(T, E);
  GemmParams p{};
  Problem& P = p.pr[0];
  if (!make_map(&P.a_s, h, T, D, BM) || !make_map(&P.b0_s, wr3, E, 3ull * D, bn)) {
    *why = "cuTensorMapEncodeTiled failed for a router operand";
    return cudaErrorInvalidValue;
  }
  P.a_r = P.a_s;
  P.b0_r = P.b1_r = P.b1_s = P.b0_s;
  P.out_r = nullptr;
  P.out_s = partials;
  P.K_r = 0; P.K_s = 3 * D;
  P.N_r = 0; P.N_s = E;
  P.a_s_group_stride = 0;
  P.b_r_group_rows = 0;
  P.b_s_group_rows = 0;
  P.bn_out = bn;
  P.k_chunk = chunk;
  P.a_k_mod = D;
  P.gateup = 0;
  p.offsets = nullptr;
  p.status = nullptr;
  p.counters = nullptr;
  p.nprob = 1;
  p.E = 0; p.S = nsplit; p.T = T;
  p.rows_r = 0;
  const int tiles = nsplit * ((T + BM - 1) / BM) * ((E + bn - 1) / bn);
  return bn == 128 ? launch_one<128>(p, tiles, st) : launch_one<256>(p, tiles, st);
}

// Small batches (T <= 512) leave each expert with at most a few row tiles, so
// the weight stream is the whole cost: 128-wide tiles double the tile count
// and keep every SM streaming.  Larger batches use 256-wide tiles.
bool use_narrow_tiles(int T) { return T <= 512; }

cudaError_t launch_expert_ffn(const FfnArgs& a, cudaStream_t st, int* nlaunch, const char** why,
                              void* const* marks) {
  const int rows_r = a.T * a.k;
  const int mt_upper = (rows_r + BM - 1) / BM + a.E;  // sum over experts of ceil(count/BM)
  const int mt_s = (a.T + BM - 1) / BM;
  const bool narrow = use_narrow_tiles(a.T);
  const int nmma = narrow ? 128 : 256;
  const int half = nmma / 2;

  GemmParams p{};
  // ---- problem 0: gate/up ----
  Problem& G = p.pr[0];
  bool ok = make_map(&G.a_r, a.xperm, rows_r, a.D, BM) &&
            make_map(&G.b0_r, a.W1, (uint64_t)a.E * a.F, a.D, half) &&
            make_map(&G.b1_r, a.W3, (uint64_t)a.E * a.F, a.D, half);
  if (ok && a.S > 0)
    ok = make_map(&G.a_s, a.h, a.T, a.D, BM) &&
         make_map(&G.b0_s, a.Ws1, (uint64_t)a.S * a.Fs, a.D, half) &&
         make_map(&G.b1_s, a.Ws3, (uint64_t)a.S * a.Fs, a.D, half);
  // ---- problem 1: down ----
  Problem& Dn = p.pr[1];
  ok = ok && make_map(&Dn.a_r, a.act_r, rows_r, a.F, BM) &&
       make_map(&Dn.b0_r, a.W2, (uint64_t)a.E * a.D, a.F, nmma);
  if (ok && a.S > 0)
    ok = make_map(&Dn.a_s, a.act_s, (uint64_t)a.S * a.T, a.Fs, BM) &&
         make_map(&Dn.b0_s, a.Ws2, (uint64_t)a.S * a.D, a.Fs, nmma);
  if (!ok) {
    *why = "cuTensorMapEncodeTiled failed for an expert operand";
    return cudaErrorInvalidValue;
  }
  G.out_r = a.act_r;
  G.out_s = a.act_s;
  G.K_r = a.D; G.K_s = a.D;
  G.N_r = a.F; G.N_s = a.Fs;
  G.a_s_group_stride = 0;
  G.b_r_group_rows = a.F;
  G.b_s_group_rows = a.Fs;
  G.bn_out = half;
  G.k_chunk = 0;
  G.a_k_mod = 0;
  G.gateup = 1;

  Dn.b1_r = Dn.b0_r;
  Dn.b1_s = Dn.b0_s;
  Dn.out_r = a.y;
  Dn.out_s = a.y + (size_t)rows_r * a.D;
  Dn.K_r = a.F; Dn.K_s = a.Fs;
  Dn.N_r = a.D; Dn.N_s = a.D;
  Dn.a_s_group_stride = a.T;
  Dn.b_r_group_rows = a.D;
  Dn.b_s_group_rows = a.D;
  Dn.bn_out = nmma;
  Dn.k_chunk = 0;
  Dn.a_k_mod = 0;
  Dn.gateup = 0;

  p.offsets = a.offsets;
  p.status = a.status;
  p.counters = a.counters;
  p.nprob = 2;
  p.E = a.E; p.S = a.S; p.T = a.T;
  p.rows_r = rows_r;
  const int tiles_g = mt_upper * ((a.F + half - 1) / half) + a.S * mt_s * ((a.Fs + half - 1) / half);
  const int nt_d = (a.D + nmma - 1) / nmma;
  const int tiles_d = mt_upper * nt_d + a.S * mt_s * nt_d;
  cudaError_t err = narrow ? launch_one<128>(p, tiles_g + tiles_d, st)
                           : launch_one<256>(p, tiles_g + tiles_d, st);
  if (err == cudaSuccess && marks) err = cudaEventRecord(static_cast<cudaEvent_t>(marks[0]), st);
  *nlaunch += 1;
  return err;
}

}  // namespace moe
