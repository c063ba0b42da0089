// Expert FFN for large batches on SM pairs: tcgen05.mma.cta_group::2 with the
// weights as the 256-row operand and the tokens as the N operand.
//
// The layer is the bf16 kernel's (grouped_gemm.cu): per routed expert on the
// rows grouped to it, and per shared expert on every token,
//   act = silu(x W1^T) * (x W3^T)      y = act W2^T
// ("GLM-5.2", PocketLLM, Implemented execution path, names w1/w3 and w2;
// "Model anatomy -- GLM-5.2", MoE panel, for the routed/shared split).  Only
// the tiling differs, for batches whose experts hold many rows each:
//   * two CTAs on a pair of SMs (a cluster of two) run one 256-row MMA: each
//     CTA stages its own 128 weight rows and half of the token rows in its own
//     shared memory and keeps its 128 rows of the accumulator in its own TMEM,
//     so each SM reads half the shared-memory bytes per multiply-add that a
//     one-SM 128 x 256 tile needs;
//   * the token rows of one expert are the MMA's N (at most 256, rounded up to
//     16), so an expert of 200 rows costs 208 columns of tensor work, where
//     128-row token tiles would cost 256 rows.
// Tiles (the D^T = W . X^T form: TMEM lanes are output features, columns are
// tokens):
//   gate/up  one group x one block of 256 tokens x 128 features: CTA r stages
//            W1 and W3 rows of features [64r, 64r + 64) of the block,
//            interleaved 16 rows at a time, so that TMEM lane quarter q of
//            each CTA holds gate (lanes 0-15) and up (lanes 16-31) of the
//            same 16 features and the epilogue pairs them with one shuffle;
//   down     one group x one block of 256 tokens x 256 output columns: CTA r
//            stages W2 rows [128r, 128r + 128) of the block.
// Tiles are numbered as in the bf16 kernel (gate/up first, down after;
// routed groups expert-major with the token block fastest, then the shared
// groups).  The pair claims every tile from the workspace counter, so tiles
// go only to running pairs, and a down tile of a group waits until both CTAs'
// epilogues of every gate/up tile of that group have stored their rows
// (bounded acquire waits on per-group counters).
//
// CTA (224 threads, one CTA per SM, two CTAs per cluster; rank 0 leads):
//   warp 6     weight producer: TMA of its 128 weight rows into an 8-stage ring
//              of its own shared memory; never waits for the gate/up -> down
//              hand-off, so the weight stream (read from HBM, once per token
//              block) runs ahead of the tokens.  The leader's also claims the
//              tiles and writes each one into both CTAs' tile queues.
//   warp 0     token producer: TMA of its half of the tile's token rows into a
//              4-stage ring (they come from L2); waits for the hand-off before
//              a down tile.  A token stage is free again once the MMAs of the
//              K-block four back have completed, read off that K-block's
//              weight-stage barrier (the weight ring is the deeper one).
//              The loads of both CTAs signal the leader's "full" barriers,
//              which expect the bytes of both.
//   warp 1     TMEM allocator (512 columns, both CTAs).  In the leader: the
//              MMA issuer (M = 256, N = tokens, K = 16, fp32 accumulators, two
//              buffers), committing each K-block to both CTAs' weight-stage
//              "empty" barriers and each finished accumulator to both CTAs'
//              epilogues.
//   warps 2-5  epilogue: tcgen05.ld of its TMEM lane quarter, SiLU gate and
//              bf16 stores (gate/up) or fp32 stores (down).
// Every wait is bounded (about a second); a timeout raises the CTA's abort
// flag, the roles unwind, and MOE_ERR_TIMEOUT is reported.
#include <cuda_bf16.h>

#include "ffn_common.cuh"

namespace moe {
namespace {

using namespace ffn;

constexpr int TB = 256;                         // token block: the MMA's N is at most 256
constexpr int W_ROWS = 128;                     // weight rows per CTA (M = 256 per pair)
constexpr int GU_BOX = 16;                      // gate/up weight rows per TMA box
constexpr int TOK_BOX = 32;                     // token rows per TMA box
constexpr int W_STAGES = 8;                     // weight ring (HBM latency)
constexpr int T_STAGES = 4;                     // token ring (L2 latency)
constexpr int A_STAGE = W_ROWS * BK * 2;        // 16 KiB of weights
constexpr int B_STAGE = (TB / 2) * BK * 2;      // 16 KiB: this CTA's half of the tokens
constexpr int TOK_BOX_BYTES = TOK_BOX * BK * 2; // 4 KiB
constexpr int GU_BOX_BYTES = GU_BOX * BK * 2;   // 2 KiB
constexpr int THREADS = 224;
constexpr int TPROD_WARP = 0;                   // token producer
constexpr int WPROD_WARP = 6;                   // weight producer (and, in the leader, claimer)
constexpr int MMA_WARP = 1;                     // TMEM allocator; MMA issuer in the leader
constexpr uint32_t TMEM_COLS = 512;             // two accumulator buffers of 256 columns
constexpr uint32_t ACC_COLS = 256;
// Tile-queue consumers that release a slot: leader token producer, MMA issuer
// and 4 epilogue warps; other CTA: weight producer, token producer and 4
// epilogue warps.
constexpr int TQ_RELEASES = 12;
constexpr uint16_t BOTH = 0x3;                  // multicast mask: both CTAs of the pair

static_assert(A_STAGE % 1024 == 0 && B_STAGE % 1024 == 0, "stages stay 1024-byte aligned");
// The token producer reuses a token stage once the MMAs of the K-block
// T_STAGES earlier have completed, which it reads off that K-block's
// weight-stage barrier; with W_STAGES >= T_STAGES that barrier cannot have
// moved on by a further phase before the producer looks.
static_assert(W_STAGES >= T_STAGES, "token stages are released through the weight ring");
static_assert(4 * 2 * GU_BOX_BYTES == A_STAGE, "8 gate/up boxes fill a weight stage");

struct PairState {
  uint64_t wfull[W_STAGES];     // leader: both CTAs' weight bytes of the stage landed
  uint64_t wempty[W_STAGES];    // the K-block's MMAs completed (leader's commit, both CTAs)
  uint64_t tfull[T_STAGES];     // leader: both CTAs' token bytes of the stage landed
  uint64_t tq_full[TILE_Q], tq_empty[TILE_Q];
  int tq_tile[TILE_Q];
  uint64_t tmem_full[2];        // accumulator ready (leader's commit, both CTAs)
  uint64_t tmem_empty[2];       // leader: both CTAs' epilogues read the accumulator
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
  TileMap tm;
};

// MMA N of a tile: its token rows rounded up to 16 (at most TB).
__device__ __forceinline__ int tile_n(const TileInfo& ti) {
  const int r = min(TB, ti.rows - ti.m0);
  return (r + 15) & ~15;
}

// Count a down tile's group reaches once every gate/up tile of the group has
// been stored by the four epilogue warps of both CTAs.
__device__ __forceinline__ int pair_rows_ready_target(const GemmParams& p, const TileInfo& ti) {
  return 2 * rows_ready_target(p, ti);
}

__global__ void __launch_bounds__(THREADS, 1) pair_ffn_kernel(const __grid_constant__ GemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = ptx::smem_addr(smem_raw);
  uint8_t* ring_a = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);   // weights
  uint8_t* ring_b = ring_a + W_STAGES * A_STAGE;                               // tokens
  PairState& ss = *reinterpret_cast<PairState*>(ring_b + T_STAGES * B_STAGE);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = ptx::cluster_ctarank();
  const bool leader = rank == 0;

  ptx::pdl_launch_dependents();
  if (threadIdx.x == 0) {
    for (int i = 0; i < W_STAGES; ++i) {
      ptx::mbar_init(&ss.wfull[i], 1);
      ptx::mbar_init(&ss.wempty[i], 1);
    }
    for (int i = 0; i < T_STAGES; ++i) ptx::mbar_init(&ss.tfull[i], 1);
    for (int i = 0; i < TILE_Q; ++i) {
      ptx::mbar_init(&ss.tq_full[i], 1);
      ptx::mbar_init(&ss.tq_empty[i], TQ_RELEASES);
    }
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(&ss.tmem_full[i], 1);
      ptx::mbar_init(&ss.tmem_empty[i], 2 * EPI_WARPS);
    }
    ptx::mbar_init(&ss.drain, 1);
    ss.abort = 0;
    ptx::fence_barrier_init();
  }
  if (warp == MMA_WARP) {
    ptx::tmem_alloc_pair(&ss.tmem_base, TMEM_COLS);
    ptx::tmem_relinquish_pair();
  }
  if (warp == TPROD_WARP && lane == 0) {
    ptx::tma_prefetch_desc(&p.pr[0].a_r);
  } else if (warp == WPROD_WARP && lane == 0) {
    ptx::tma_prefetch_desc(&p.pr[0].b0_r);
    ptx::tma_prefetch_desc(&p.pr[0].b1_r);
  }
  // both CTAs' barriers are initialised (and TMEM allocated) before either
  // CTA touches the other's
  ptx::tc_fence_before();
  ptx::cluster_sync();
  ptx::tc_fence_after();

  // everything below reads what earlier kernels in the stream wrote
  ptx::pdl_wait();
  int first = 0;
  if (leader && warp == WPROD_WARP && lane == 0) first = first_tile(p);
  if (warp == 2) build_tile_map<TB>(ss.tm, p, lane);
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();

  const uint32_t tmem_base = ss.tmem_base;
  const int tiles0 = problem_tiles<TB>(p.pr[0], ss.tm, p);
  const int total = tiles0 + (p.nprob > 1 ? problem_tiles<TB>(p.pr[1], ss.tm, p) : 0);
  volatile int* abort = &ss.abort;
  const uint32_t peer = rank ^ 1u;

  // A consumer takes the tile in queue slot `qslot` and releases the slot to
  // the leader's producer.
  auto take_tile = [&](int qslot, uint32_t qphase, int* tile) -> bool {
    if (!ptx::mbar_wait_cluster(&ss.tq_full[qslot], qphase, abort)) return false;
    *tile = *reinterpret_cast<volatile int*>(&ss.tq_tile[qslot]);
    if (leader)
      ptx::mbar_arrive(&ss.tq_empty[qslot]);
    else
      ptx::mbar_arrive_cluster(ptx::map_to_rank(ptx::smem_addr(&ss.tq_empty[qslot]), 0));
    return true;
  };

  if (warp == WPROD_WARP) {
    // ---------------- weight producer (both CTAs); the leader's also claims ----------------
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued = 0, last_par = 0;
      int qslot = 0;
      uint32_t qphase = 0;
      int tile = first;
      int next = 0;
      if (leader) next = tile < total ? claim_tile(p, tile) : total;
      for (;;) {
        if (leader) {
          // publish the tile (or the end mark) to both CTAs' queues
          if (!ptx::mbar_wait_cluster(&ss.tq_empty[qslot], qphase ^ 1u, abort)) break;
          const int v = tile < total ? tile : -1;
          ss.tq_tile[qslot] = v;
          ptx::st_cluster_u32(ptx::map_to_rank(ptx::smem_addr(&ss.tq_tile[qslot]), peer),
                              (uint32_t)v);
          ptx::mbar_arrive_cluster(ptx::map_to_rank(ptx::smem_addr(&ss.tq_full[qslot]), peer));
          ptx::mbar_arrive(&ss.tq_full[qslot]);
          if (++qslot == TILE_Q) { qslot = 0; qphase ^= 1u; }
          if (v < 0) break;
        } else {
          if (!take_tile(qslot, qphase, &tile)) break;
          if (++qslot == TILE_Q) { qslot = 0; qphase ^= 1u; }
          if (tile < 0) break;
        }
        const TileInfo ti = decode_tile<TB>(tile, ss.tm, p, tiles0);
        const Problem& P = p.pr[ti.prob];
        const CUtensorMap* b0 = ti.shared ? &P.b0_s : &P.b0_r;
        const CUtensorMap* b1 = ti.shared ? &P.b1_s : &P.b1_r;
        const int grp_rows = ti.shared ? P.b_s_group_rows : P.b_r_group_rows;
        // gate/up: features [n0 + 64r, n0 + 64r + 64); down: W2 rows [n0 + 128r, +128)
        const int w_row = ti.grp * grp_rows + ti.n0 + (int)rank * (P.gateup ? 64 : W_ROWS);
        int kbeg, K;
        tile_k_range(ti, P, &kbeg, &K);
        const int nk = (K + BK - 1) / BK;
        bool ok = true;
        for (int kb = 0; kb < nk; ++kb) {
          if (!ptx::mbar_wait(&ss.wempty[stage], phase ^ 1u, abort)) { ok = false; break; }
          uint8_t* sa = ring_a + stage * A_STAGE;
          const int x = kbeg + kb * BK;
          const uint32_t fb = ptx::map_to_rank(ptx::smem_addr(&ss.wfull[stage]), 0);
          // the leader's barrier counts the weight bytes of both CTAs
          if (leader) ptx::mbar_arrive_expect_tx(&ss.wfull[stage], 2 * A_STAGE);
          if (P.gateup) {
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              ptx::tma_load_2d_pair(sa + q * 2 * GU_BOX_BYTES, b0, fb, x, w_row + q * GU_BOX);
              ptx::tma_load_2d_pair(sa + q * 2 * GU_BOX_BYTES + GU_BOX_BYTES, b1, fb, x,
                                    w_row + q * GU_BOX);
            }
          } else {
            ptx::tma_load_2d_pair(sa, b0, fb, x, w_row);
          }
          issued |= 1u << stage;
          last_par = (last_par & ~(1u << stage)) | (phase << stage);
          if (++stage == W_STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        if (leader) {
          tile = next;
          next = tile < total ? claim_tile(p, tile) : total;
        }
      }
      // Every load issued has landed before the pair may retire: the leader
      // waits for the last phase of each stage it filled, which counts the
      // other CTA's bytes of that phase too (both producers fill the same
      // stages in the same order); the other CTA retires only after the
      // leader, at the final cluster barrier.
      if (leader)
        for (int s = 0; s < W_STAGES; ++s)
          if (issued & (1u << s)) wait_drain(&ss.wfull[s], (last_par >> s) & 1u, abort);
    }
  } else if (warp == TPROD_WARP) {
    // ---------------- token producer (both CTAs) ----------------
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued = 0, last_par = 0;
      // position, in the weight ring, of the K-block T_STAGES behind this one
      int rstage = 0;
      uint32_t rphase = 0;
      int lag = T_STAGES;   // K-blocks still to go before that position exists
      int qslot = 0;
      uint32_t qphase = 0;
      for (;;) {
        int tile;
        if (!take_tile(qslot, qphase, &tile)) break;
        if (++qslot == TILE_Q) { qslot = 0; qphase ^= 1u; }
        if (tile < 0) break;
        const TileInfo ti = decode_tile<TB>(tile, ss.tm, p, tiles0);
        const Problem& P = p.pr[ti.prob];
        if (ti.prob == 1) {
          // this tile's activations come from the group's gate/up epilogues
          const int g = ti.shared ? p.E + ti.grp : ti.grp;
          if (!ptx::counter_wait(p.counters + g, pair_rows_ready_target(p, ti), abort)) break;
          ptx::fence_proxy_async_global();
        }
        const CUtensorMap* amap = ti.shared ? &P.a_s : &P.a_r;
        const int half = tile_n(ti) / 2;             // this CTA's token rows
        const int nbox = (half + TOK_BOX - 1) / TOK_BOX;
        const int a_row = (ti.shared ? ti.grp * P.a_s_group_stride + ti.m0 : ti.row0 + ti.m0) +
                          (int)rank * half;
        int kbeg, K;
        tile_k_range(ti, P, &kbeg, &K);
        const int nk = (K + BK - 1) / BK;
        bool ok = true;
        for (int kb = 0; kb < nk; ++kb) {
          // the stage's previous K-block (T_STAGES back) has finished its MMAs
          if (lag > 0) {
            --lag;
          } else {
            if (!ptx::mbar_wait(&ss.wempty[rstage], rphase, abort)) { ok = false; break; }
            if (++rstage == W_STAGES) { rstage = 0; rphase ^= 1u; }
          }
          uint8_t* sb = ring_b + stage * B_STAGE;
          const int x = kbeg + kb * BK;
          const uint32_t fb = ptx::map_to_rank(ptx::smem_addr(&ss.tfull[stage]), 0);
          if (leader) ptx::mbar_arrive_expect_tx(&ss.tfull[stage], 2 * nbox * TOK_BOX_BYTES);
          for (int b = 0; b < nbox; ++b)
            ptx::tma_load_2d_pair(sb + b * TOK_BOX_BYTES, amap, fb, x, a_row + b * TOK_BOX);
          issued |= 1u << stage;
          last_par = (last_par & ~(1u << stage)) | (phase << stage);
          if (++stage == T_STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
      }
      if (leader)
        for (int s = 0; s < T_STAGES; ++s)
          if (issued & (1u << s)) wait_drain(&ss.tfull[s], (last_par >> s) & 1u, abort);
    }
  } else if (warp == MMA_WARP) {
    if (lane == 0 && leader) {
      // ---------------- MMA issuer (leader) ----------------
      int wstage = 0, tstage = 0;
      uint32_t wphase = 0, tphase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      int qslot = 0;
      uint32_t qphase = 0;
      for (;;) {
        int tile;
        if (!take_tile(qslot, qphase, &tile)) break;
        if (++qslot == TILE_Q) { qslot = 0; qphase ^= 1u; }
        if (tile < 0) break;
        const TileInfo ti = decode_tile<TB>(tile, ss.tm, p, tiles0);
        int kbeg, K;
        tile_k_range(ti, p.pr[ti.prob], &kbeg, &K);
        const int nk = (K + BK - 1) / BK;
        const uint32_t idesc = ptx::idesc_bf16_f32(2 * W_ROWS, tile_n(ti));
        if (!ptx::mbar_wait_cluster(&ss.tmem_empty[acc], acc_phase ^ 1u, abort)) break;
        ptx::tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * ACC_COLS;
        bool ok = true;
        uint32_t accumulate = 0;
        for (int kb = 0; kb < nk; ++kb) {
          if (!ptx::mbar_wait(&ss.wfull[wstage], wphase, abort) ||
              !ptx::mbar_wait(&ss.tfull[tstage], tphase, abort)) {
            ok = false;
            break;
          }
          ptx::tc_fence_after();
          // descriptor start-address fields count 16-byte units: +2 per K step
          const uint64_t a_desc = ptx::smem_desc_sw128(ptx::smem_addr(ring_a + wstage * A_STAGE));
          const uint64_t b_desc = ptx::smem_desc_sw128(ptx::smem_addr(ring_b + tstage * B_STAGE));
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            ptx::mma_pair_f16_ss(d_tmem, a_desc + 2 * kk, b_desc + 2 * kk, idesc, accumulate);
            accumulate = 1;
          }
          // frees the weight stage in both CTAs, and the token stage to the
          // token producers' next lap, when these MMAs finish
          ptx::mma_commit_pair_mc(&ss.wempty[wstage], BOTH);
          if (++wstage == W_STAGES) { wstage = 0; wphase ^= 1u; }
          if (++tstage == T_STAGES) { tstage = 0; tphase ^= 1u; }
        }
        if (!ok) break;
        ptx::mma_commit_pair_mc(&ss.tmem_full[acc], BOTH);   // both CTAs' epilogues
        if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
      }
      ptx::mma_commit_pair(&ss.drain);
      wait_drain(&ss.drain, 0, abort);
    }
  } else {
    // ---------------- epilogue (warps 2..5, both CTAs) ----------------
    const int q = warp & 3;   // TMEM lane quarter this warp may access
    int acc = 0;
    uint32_t acc_phase = 0;
    int qslot = 0;
    uint32_t qphase = 0;
    for (;;) {
      int tile = -1;
      bool got = true;
      if (lane == 0) got = take_tile(qslot, qphase, &tile);
      got = __shfl_sync(0xffffffffu, got ? 1 : 0, 0) != 0;
      tile = __shfl_sync(0xffffffffu, tile, 0);
      if (!got) break;
      if (++qslot == TILE_Q) { qslot = 0; qphase ^= 1u; }
      if (tile < 0) break;
      const TileInfo ti = decode_tile<TB>(tile, ss.tm, p, tiles0);
      const Problem& P = p.pr[ti.prob];
      const int ncols = tile_n(ti);
      if (!ptx::mbar_wait(&ss.tmem_full[acc], acc_phase, abort)) break;
      ptx::tc_fence_after();
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + acc * ACC_COLS;
      const int N = ti.shared ? P.N_s : P.N_r;
      const int valid = ti.rows - ti.m0;      // token rows of this block
      if (P.gateup) {
        uint16_t* out = static_cast<uint16_t*>(ti.shared ? P.out_s : P.out_r);
        const int f = ti.n0 + (int)rank * 64 + q * 16 + (lane & 15);
        const bool f_ok = f < N;
        const bool up_half = lane >= 16;
#pragma unroll 1
        for (int c = 0; c < ncols; c += 16) {
          uint32_t v[16];
          ptx::tmem_ld_x16(taddr + c, v);
          ptx::tmem_wait_ld();
          // lanes 0-15 hold gate rows, lanes 16-31 the up rows of the same
          // features: lane l < 16 finishes tokens c..c+7, lane l + 16 tokens
          // c+8..c+15 of feature f
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const uint32_t send = up_half ? v[j] : v[8 + j];
            const float other = __uint_as_float(__shfl_xor_sync(0xffffffffu, send, 16));
            const float g = up_half ? other : __uint_as_float(v[j]);
            const float u = up_half ? __uint_as_float(v[8 + j]) : other;
            const int tok = c + (up_half ? 8 : 0) + j;
            if (f_ok && tok < valid) {
              const __nv_bfloat16 a = __float2bfloat16_rn(silu_times(g, u));
              out[(size_t)(ti.row0 + ti.m0 + tok) * N + f] = __bfloat16_as_ushort(a);
            }
          }
        }
      } else {
        float* out = static_cast<float*>(ti.shared ? P.out_s : P.out_r);
        const int dcol = ti.n0 + (int)rank * W_ROWS + q * 32 + lane;
        const bool d_ok = dcol < N;
#pragma unroll 1
        for (int c = 0; c < ncols; c += 16) {
          uint32_t v[16];
          ptx::tmem_ld_x16(taddr + c, v);
          ptx::tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 16; ++j)
            if (d_ok && c + j < valid)
              out[(size_t)(ti.row0 + ti.m0 + c + j) * N + dcol] = __uint_as_float(v[j]);
        }
      }
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (leader)
          ptx::mbar_arrive(&ss.tmem_empty[acc]);
        else
          ptx::mbar_arrive_cluster(ptx::map_to_rank(ptx::smem_addr(&ss.tmem_empty[acc]), 0));
      }
      if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
      if (p.nprob > 1 && ti.prob == 0) release_rows(p, ti, lane);
    }
  }

  // Both CTAs retire together: the leader's MMAs (which read the other CTA's
  // shared memory) have drained and both epilogues are done with TMEM.
  ptx::tc_fence_before();
  __syncthreads();
  ptx::cluster_sync();
  if (warp == MMA_WARP) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc_pair(tmem_base, TMEM_COLS);
  }
  if (threadIdx.x == 0 && ss.abort && p.status) atomicOr(p.status, kStTimeout);
}

constexpr size_t kSmemBytes = 1024 + W_STAGES * A_STAGE + T_STAGES * B_STAGE + sizeof(PairState);
static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");

bool make_map_rows(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols,
                   uint32_t box_rows) {
  return make_tensor_map(m, base, rows, cols, box_rows, BK, 2, 128);
}

// Pairs that fit on the device at once (cached per device).
int max_pairs(const cudaLaunchConfig_t& cfg) {
  static int cache[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && cache[dev] > 0) return cache[dev];
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, pair_ffn_kernel, &cfg) != cudaSuccess || n < 1) {
    cudaGetLastError();
    n = num_sms() / 2;
  }
  if (dev >= 0 && dev < 64) cache[dev] = n;
  return n;
}

}  // namespace

bool use_pair_ffn(int T) { return T > 512; }

cudaError_t launch_expert_ffn_pair(const FfnArgs& a, cudaStream_t st, int* nlaunch,
                                   const char** why, void* const* marks) {
  const int rows_r = a.T * a.k;
  GemmParams p{};
  // ---- problem 0: gate/up (weights as the 256-row operand) ----
  Problem& G = p.pr[0];
  bool ok = make_map_rows(&G.a_r, a.xperm, rows_r, a.D, TOK_BOX) &&
            make_map_rows(&G.b0_r, a.W1, (uint64_t)a.E * a.F, a.D, GU_BOX) &&
            make_map_rows(&G.b1_r, a.W3, (uint64_t)a.E * a.F, a.D, GU_BOX);
  if (ok && a.S > 0)
    ok = make_map_rows(&G.a_s, a.h, a.T, a.D, TOK_BOX) &&
         make_map_rows(&G.b0_s, a.Ws1, (uint64_t)a.S * a.Fs, a.D, GU_BOX) &&
         make_map_rows(&G.b1_s, a.Ws3, (uint64_t)a.S * a.Fs, a.D, GU_BOX);
  // ---- problem 1: down ----
  Problem& Dn = p.pr[1];
  ok = ok && make_map_rows(&Dn.a_r, a.act_r, rows_r, a.F, TOK_BOX) &&
       make_map_rows(&Dn.b0_r, a.W2, (uint64_t)a.E * a.D, a.F, W_ROWS);
  if (ok && a.S > 0)
    ok = make_map_rows(&Dn.a_s, a.act_s, (uint64_t)a.S * a.T, a.Fs, TOK_BOX) &&
         make_map_rows(&Dn.b0_s, a.Ws2, (uint64_t)a.S * a.D, a.Fs, W_ROWS);
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
  G.bn_out = W_ROWS;            // 128 features per pair tile
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
  Dn.bn_out = 2 * W_ROWS;       // 256 output columns per pair tile
  Dn.gateup = 0;

  p.offsets = a.offsets;
  p.status = a.status;
  p.counters = a.counters;
  p.sched = a.counters + a.E + a.S;   // zeroed with the group counters
  p.weights_once = 0;
  p.nprob = 2;
  p.E = a.E; p.S = a.S; p.T = a.T;
  p.rows_r = rows_r;

  // tiles: an upper bound for sizing the grid
  const int mt_r = (rows_r + TB - 1) / TB + a.E;
  const int mt_s = (a.T + TB - 1) / TB;
  const int tiles = mt_r * ((a.F + W_ROWS - 1) / W_ROWS) +
                    a.S * mt_s * ((a.Fs + W_ROWS - 1) / W_ROWS) +
                    (mt_r + a.S * mt_s) * ((a.D + 2 * W_ROWS - 1) / (2 * W_ROWS));

  static int configured_dev = -1;
  int dev = 0;
  cudaGetDevice(&dev);
  if (configured_dev != dev) {
    cudaError_t e = cudaFuncSetAttribute(pair_ffn_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kSmemBytes);
    if (e != cudaSuccess) {
      *why = "pair FFN shared memory attribute";
      return e;
    }
    configured_dev = dev;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(THREADS);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cfg.gridDim = dim3(2);
  int pairs = max_pairs(cfg);
  if (tiles < pairs) pairs = tiles;
  if (pairs < 1) pairs = 1;
  cfg.gridDim = dim3(2 * pairs);
  cfg.numAttrs = 2;
  cudaError_t err = cudaLaunchKernelEx(&cfg, pair_ffn_kernel, p);
  if (err != cudaSuccess) *why = "pair FFN launch";
  if (err == cudaSuccess && marks) err = cudaEventRecord(static_cast<cudaEvent_t>(marks[0]), st);
  *nlaunch += 1;
  return err;
}

}  // namespace moe
