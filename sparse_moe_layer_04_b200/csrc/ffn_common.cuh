// Pieces shared by the expert-FFN kernels (bf16 weights in grouped_gemm.cu,
// FP8 weights in ffn_fp8.cu) and the tensor-core router: the grouped-problem
// description, the device-side tile map built from the group offsets, tile
// decoding, and small epilogue helpers.
#pragma once

#include <cuda_bf16.h>

#include "moe_internal.cuh"
#include "sm100_ptx.cuh"

namespace moe {
namespace ffn {

constexpr int BM = 128;
constexpr int BK = 64;                    // one 128-byte swizzle row of bf16
constexpr int A_BYTES = BM * BK * 2;      // 16 KiB
constexpr int MAX_E = 1024;
constexpr int EPI_WARPS = 4;              // each releases its rows of a gate/up tile
constexpr unsigned kWarpMask = 0xffffffffu;

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
  // FP8 weights only: int8 block exponents of b0/b1 (routed, shared), laid out
  // [group][row block][K block] with `rb` row blocks per group and `kb` K blocks
  const int8_t* e0_r;
  const int8_t* e1_r;
  const int8_t* e0_s;
  const int8_t* e1_s;
  int rb_r, rb_s, kb_r, kb_s;
};

struct GemmParams {
  Problem pr[2];
  const int32_t* offsets;    // [E+1] routed group row offsets (E > 0)
  int* status;
  int* counters;             // [E+S] gate/up tiles stored per group (two problems)
  int* sched;                // tile claim counter, zero at launch; nullptr: static round-robin
  int* exit_ticket;          // nullable: the CTA that takes the last ticket at exit zeroes
  int nreset;                // `counters[0, nreset)`, the claim counter and the ticket
  int weights_once;          // 1: weight tiles are read by about one row tile each, so
                             // they are loaded with an L2 evict-first policy
  int nprob;                 // 1 or 2
  int E, S, T;
  int rows_r;                // T * k
  // Batches of at most 128 tokens (one row tile): the A operand of every
  // routed gate/up tile is the whole token matrix (a_r maps h [T, D]), so no
  // gathered copy is made, and the epilogue writes the row of each token
  // routed to the tile's expert at that pair's grouped row (from idx / inv);
  // the other tokens' rows are dropped.
  int dense_a;
  int k;
  const int32_t* idx;        // [T, k] (dense_a)
  const int32_t* inv;        // [T, k] (dense_a)
  // Batches of at most 128 tokens routed without a grouping pass: `mask`
  // [E][mask_stride] holds bit t of row e when token t chose expert e (rows
  // of ceil(T / 32) words).  The group row offsets are then those of the
  // pairs in (expert, token) order: each CTA derives them from the bit
  // counts, CTA 0 also stores counts [E], offsets [E + 1] and the number of
  // experts with pairs (touched), and the gate/up epilogue writes inv for
  // the pairs it places.  nullptr: offsets come from `offsets`.
  const uint32_t* mask;
  int mask_stride;
  int32_t* counts_out;
  int32_t* offsets_out;
  int32_t* touched_out;
  int32_t* inv_out;
};

// Row blocks of the routed groups, built on the device from the group
// offsets.  A row block is BR rows of a group (BM = 128 for the bf16 kernel,
// the token block for the FP8 kernel).
struct TileMap {
  int mt_total;              // routed row blocks over all experts
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

// Token-bit mode (GemmParams::mask): rows of at most kMaskWords words (T <=
// 128), read kMaskBatch chunks of 32 experts at a time.
constexpr int kMaskWords = 4;
constexpr int kMaskBatch = 8;

// One warp reads the group offsets (or counts the token bits) 32 experts at
// a time, checks them and writes the row-tile prefix; inconsistent offsets
// give an empty routed tile space and raise kStBounds.
template <int BR = BM>
__device__ __forceinline__ void build_tile_map(TileMap& tm, const GemmParams& p, int lane) {
  int carry = 0;
  bool bad = false;
  if (p.mask) {
    // token bits (T <= 128: at most kMaskWords words per expert row): the
    // rows of kMaskBatch chunks of 32 experts are loaded together, then
    // scanned chunk by chunk
    int row_carry = 0, touched = 0;
    const int words = (p.T + 31) >> 5;
    const bool store = blockIdx.x == 0;
    for (int base0 = 0; base0 < p.E; base0 += 32 * kMaskBatch) {
      uint32_t m[kMaskBatch][kMaskWords];
#pragma unroll
      for (int c = 0; c < kMaskBatch; ++c) {
        const int e = base0 + 32 * c + lane;
#pragma unroll
        for (int q = 0; q < kMaskWords; ++q)
          m[c][q] = (e < p.E && q < words) ? p.mask[(size_t)e * p.mask_stride + q] : 0u;
      }
#pragma unroll
      for (int c = 0; c < kMaskBatch; ++c) {
        const int e = base0 + 32 * c + lane;
        int rows = 0;
#pragma unroll
        for (int q = 0; q < kMaskWords; ++q) rows += __popc(m[c][q]);
        int rincl = rows, cnt = (rows + BR - 1) / BR, incl = cnt;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
          const int v = __shfl_up_sync(0xffffffffu, rincl, off);
          const int u = __shfl_up_sync(0xffffffffu, incl, off);
          if (lane >= off) {
            rincl += v;
            incl += u;
          }
        }
        if (e < p.E) {
          const int a = row_carry + rincl - rows;
          tm.off[e] = a;
          tm.mt_prefix[e] = carry + incl - cnt;
          if (store) {
            p.counts_out[e] = rows;
            p.offsets_out[e] = a;
          }
        }
        row_carry += __shfl_sync(0xffffffffu, rincl, 31);
        carry += __shfl_sync(0xffffffffu, incl, 31);
        touched += __popc(__ballot_sync(0xffffffffu, rows > 0));
      }
    }
    if (lane == 0) {
      tm.off[p.E] = row_carry;
      bad = row_carry != p.rows_r;   // every token has k distinct experts
      if (store) {
        p.offsets_out[p.E] = row_carry;
        *p.touched_out = touched;
      }
    }
  } else {
    for (int base = 0; base < p.E; base += 32) {
      const int e = base + lane;
      int cnt = 0;
      if (e < p.E) {
        const int a = p.offsets[e], b = p.offsets[e + 1];
        tm.off[e] = a;
        if (e == p.E - 1) tm.off[p.E] = b;
        if (a < 0 || b < a || b > p.rows_r || (e == 0 && a != 0)) bad = true;
        cnt = b >= a ? (b - a + BR - 1) / BR : 0;
      }
      int incl = cnt;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += v;
      }
      if (e < p.E) tm.mt_prefix[e] = carry + incl - cnt;
      carry += __shfl_sync(0xffffffffu, incl, 31);
    }
  }
  bad = __any_sync(0xffffffffu, bad);
  if (lane == 0) {
    tm.mt_prefix[p.E] = carry;
    tm.mt_total = bad ? 0 : carry;
    if (bad && p.status) atomicOr(p.status, kStBounds);
  }
}

template <int BR = BM>
__device__ __forceinline__ int problem_tiles(const Problem& P, const TileMap& tm,
                                             const GemmParams& p) {
  const int mt_s = (p.T + BR - 1) / BR;
  return tm.mt_total * col_tiles(P.N_r, P.bn_out) + p.S * mt_s * col_tiles(P.N_s, P.bn_out);
}

template <int BR = BM>
__device__ __forceinline__ TileInfo decode_tile(int tile, const TileMap& tm,
                                                const GemmParams& p, int tiles0) {
  TileInfo ti;
  ti.prob = (tile >= tiles0) ? 1 : 0;
  const Problem& P = p.pr[ti.prob];
  const int lt = tile - (ti.prob ? tiles0 : 0);
  const int nt_r = col_tiles(P.N_r, P.bn_out);
  const int routed = tm.mt_total * nt_r;
  if (lt < routed) {
    // expert e: largest with mt_prefix[e] * nt_r <= lt
    const int q = lt / nt_r;
    int lo = 0, hi = p.E - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (tm.mt_prefix[mid] <= q) lo = mid; else hi = mid - 1;
    }
    const int e = lo;
    const int rows = tm.off[e + 1] - tm.off[e];
    const int mt = (rows + BR - 1) / BR;
    const int local = lt - tm.mt_prefix[e] * nt_r;
    ti.shared = false;
    ti.grp = e;
    ti.m0 = (local % mt) * BR;
    ti.n0 = (local / mt) * P.bn_out;
    ti.rows = rows;
    ti.row0 = tm.off[e];
    ti.mt = mt;
  } else {
    const int ls = lt - routed;
    const int mt = (p.T + BR - 1) / BR;
    const int nt = col_tiles(P.N_s, P.bn_out);
    const int s = ls / (mt * nt);
    const int rem = ls - s * mt * nt;
    ti.shared = true;
    ti.grp = s;
    ti.m0 = (rem % mt) * BR;
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

// Tile scheduling.  With a claim counter (the expert FFN) a CTA claims every
// tile it runs, its first one included, from the counter, so tiles are handed
// out in increasing order and only to CTAs that are already running: a tile
// that another tile waits for (a gate/up tile of a down tile's group) is
// always held by a resident CTA, however many SMs other kernels occupy.  CTAs
// that finish early take more tiles.  Without a counter (the router GEMM,
// whose tiles wait on nothing) CTA c takes c, c + gridDim.x, ...
__device__ __forceinline__ int first_tile(const GemmParams& p) {
  return p.sched ? atomicAdd(p.sched, 1) : (int)blockIdx.x;
}
__device__ __forceinline__ int claim_tile(const GemmParams& p, int tile) {
  return p.sched ? atomicAdd(p.sched, 1) : tile + (int)gridDim.x;
}

// Leaves a launch's counters zero for the next launch that uses them: every
// CTA takes an exit ticket once all its work is done; the last one (the
// whole grid has finished its tiles) zeroes the group counters, the claim
// counter and the ticket.  Called by one thread per CTA after the final
// block-wide barrier.
__device__ __forceinline__ void reset_counters_at_exit(const GemmParams& p) {
  if (!p.exit_ticket) return;
  __threadfence();
  if (atomicAdd(p.exit_ticket, 1) == (int)gridDim.x - 1) {
    for (int i = 0; i < p.nreset; ++i) p.counters[i] = 0;
    *p.sched = 0;
    *p.exit_ticket = 0;
    __threadfence();
  }
}

// The same at block scope, called by every thread of the CTA after its final
// barrier (`s_last`: a shared int): thread 0 takes the ticket, and all
// threads of the last CTA zero the counters.
__device__ __forceinline__ void reset_counters_at_exit_block(const GemmParams& p, int* s_last) {
  if (!p.exit_ticket) return;
  if (threadIdx.x == 0) {
    __threadfence();
    *s_last = atomicAdd(p.exit_ticket, 1) == (int)gridDim.x - 1;
  }
  __syncthreads();
  if (!*s_last) return;
  __threadfence();
  for (int i = threadIdx.x; i < p.nreset; i += blockDim.x) p.counters[i] = 0;
  __syncthreads();
  if (threadIdx.x == 0) {
    *p.sched = 0;
    *p.exit_ticket = 0;
    __threadfence();
  }
}

// Queue of claimed tiles from the producer to the other roles of the CTA.
constexpr int TILE_Q = 4;

// K-blocks of a tile padded to whole rounds of `m` issuers: the padding
// stages go through the ring's barriers with no data and no MMA, so every
// tile starts on stage 0 of a round and stage s always meets issuer s % m.
__device__ __forceinline__ int round_up(int n, int m) { return (n + m - 1) / m * m; }

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

// 16 accumulator columns of this warp's lane quarter: D0, plus D1 (d1_off
// columns further) when the tile's K-blocks were split between two
// accumulators.
__device__ __forceinline__ void load_acc16(uint32_t taddr, uint32_t d1_off, bool two,
                                           uint32_t (&v)[16]) {
  ptx::tmem_ld_x16(taddr, v);
  if (two) {
    uint32_t u[16];
    ptx::tmem_ld_x16(taddr + d1_off, u);
    ptx::tmem_wait_ld();
#pragma unroll
    for (int j = 0; j < 16; ++j)
      v[j] = __float_as_uint(__uint_as_float(v[j]) + __uint_as_float(u[j]));
  } else {
    ptx::tmem_wait_ld();
  }
}

// Epilogue of one accumulator tile (warp quarter q of the four epilogue
// warps): gate/up tiles apply the SiLU gate (gate in TMEM columns [0, HALF),
// up in [HALF, 2 HALF)) and store bf16; down tiles store fp32.  `taddr` is the
// warp's TMEM lane quarter at the accumulator's first column; with `two` the
// tile is the sum of that accumulator and the one d1_off columns further.
// `row_ok` / `out_row`: whether this lane's accumulator row is stored, and
// the output row it goes to.
template <int MMA_N>
__device__ __forceinline__ void store_tile(const TileInfo& ti, const Problem& P, uint32_t taddr,
                                           uint32_t d1_off, bool two, bool row_ok,
                                           size_t out_row) {
  constexpr int HALF = MMA_N / 2;
  const int N = ti.shared ? P.N_s : P.N_r;
  if (P.gateup) {
    uint16_t* out = static_cast<uint16_t*>(ti.shared ? P.out_s : P.out_r);
#pragma unroll 1
    for (int c = 0; c < HALF; c += 16) {
      uint32_t g[16], u[16];
      load_acc16(taddr + c, d1_off, two, g);
      load_acc16(taddr + HALF + c, d1_off, two, u);
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
      load_acc16(taddr + c, d1_off, two, v);
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
}

// Releases a stored gate/up tile's rows to the down tiles of its group (one
// count per epilogue warp): the stores become visible to the async proxy and
// to the whole GPU before the count.
__device__ __forceinline__ void release_rows(const GemmParams& p, const TileInfo& ti, int lane) {
  ptx::fence_proxy_async_global();
  __threadfence();
  __syncwarp();
  if (lane == 0) atomicAdd(p.counters + (ti.shared ? p.E + ti.grp : ti.grp), 1);
}

// Count the down tiles of a tile's group wait for before reading its
// activations.
__device__ __forceinline__ int rows_ready_target(const GemmParams& p, const TileInfo& ti) {
  const int nt0 = ti.shared ? col_tiles(p.pr[0].N_s, p.pr[0].bn_out)
                            : col_tiles(p.pr[0].N_r, p.pr[0].bn_out);
  return EPI_WARPS * ti.mt * nt0;
}

}  // namespace ffn

// host side (grouped_gemm.cu)
// Row-major [rows, cols] matrix of 2-byte (bf16) or 1-byte (FP8 code)
// elements, box = box_rows x box_cols elements, shared-memory swizzle of
// `swizzle_bytes` (0, 64 or 128); out-of-range box elements read as zero.
bool make_tensor_map(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols,
                     uint32_t box_rows, uint32_t box_cols, int elem_bytes, int swizzle_bytes);

}  // namespace moe
