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
// shared experts.  Every CTA claims each of its tiles, the first one
// included, in increasing order from a counter in the workspace (zeroed by the
// row-gather kernel), so CTAs that finish early take more tiles; the weight
// producer passes each claimed tile to the other roles through a small
// shared-memory queue (the router GEMM, which has no such counter, takes c,
// c + gridDim.x, ...).  A down tile of an expert waits until every gate/up
// tile of that expert has been stored: each gate/up epilogue warp releases a
// per-expert counter after a proxy fence, and the producer acquires it before
// its TMA loads read the activations.  Down tiles therefore fill the SMs that
// the tail of the gate/up tiles leaves idle.  A tile is only ever claimed by a
// CTA that is already running, and all gate/up tiles precede all down tiles,
// so every counter a CTA waits on is advanced by tiles held by running CTAs:
// the waits end even when other kernels hold some of the SMs and only part of
// the grid is resident.  They are bounded all the same.
//
// N (the MMA width) is 256 for large batches and 128 for small ones, where
// each expert has only a row tile or two and the weight stream must be cut
// finer to keep all 148 SMs busy.  The same kernel also computes the router
// logits as a dense split-K GEMM (one problem, one shared group per K chunk).
//
// CTA structure (256 threads, one CTA per SM):
//   warp 7      weight producer and tile claimer: claims the tiles, hands them
//               to the other roles, and streams the weight tiles (N x 64 bf16,
//               128-byte swizzled) into a ring of their own by TMA: 8 stages
//               for N = 128, 4 for N = 256.  It never waits for the gate/up ->
//               down hand-off, so weight loads run ahead of the activations.
//   warp 0      token / activation producer: TMA of the A tiles (128 x 64
//               bf16) into a 4-stage ring (they come from L2); waits for the
//               hand-off before a down tile.  A token stage is free again when
//               the MMAs of the K-block four back have completed, which the
//               producer reads off that K-block's weight-stage barrier.
//   warp 1      TMEM allocator (512 columns) and MMA issuer:
//               tcgen05.mma.cta_group::1.kind::f16, M = 128, N, K = 16,
//               fp32 accumulators in TMEM, two accumulator buffers so the
//               epilogue of tile i overlaps the main loop of tile i+1.  The
//               whole warp walks the issue loop and an elected lane issues.
//   warp 6      second MMA issuer for N = 128: one warp issues a tcgen05.mma
//               per ~150 cycles (measured, whatever N), longer than an
//               N = 128 MMA runs (64 cycles), so warps 1 and 6 take alternate
//               K-blocks of a tile into two accumulators of its buffer (idle
//               for N = 256).
//   warps 2-5   epilogue: tcgen05.ld of the accumulator(s) (warp w reads TMEM
//               lanes 32*(w%4) .. +31), fused activation, global stores.
#include <cuda_bf16.h>

#include "ffn_common.cuh"

namespace moe {
namespace {

using namespace ffn;

constexpr int THREADS = 256;             // warps 0-7
static_assert(kDenseMaxT <= 32 * kMaskWords, "token-bit rows of a dense batch");

constexpr int MMA_WARP1 = 6;             // second MMA issuer (N = 128)
constexpr int BPROD_WARP = 7;            // weight producer and tile claimer
constexpr int RING_BYTES = 192 * 1024;   // budget of the two operand rings
constexpr int A_STAGES = 4;              // token / activation ring (its tiles come from L2)
constexpr int MAX_B_STAGES = 8;

template <int MMA_N>
struct Shape {
  static constexpr int B_BYTES = MMA_N * BK * 2;
  // The weight ring takes what the token ring leaves: 8 stages for N = 128,
  // 4 for N = 256.  The weights stream from HBM, so the bytes a CTA keeps in
  // flight on them set the rate at which a decode batch reads its experts.
  static constexpr int B_STAGES = (RING_BYTES - A_STAGES * A_BYTES) / B_BYTES;
  static constexpr int ACC_COLS = MMA_N;                     // fp32 TMEM columns per accumulator
  // One issuing warp (elected lane) issues a tcgen05.mma every ~150 cycles,
  // longer than an N = 128 MMA executes (64): N = 128 tiles split their
  // K-blocks between two issuing warps (~105 cycles per MMA together) with an
  // accumulator each (the epilogue adds them).
  static constexpr int MMA_WARPS = MMA_N == 128 ? 2 : 1;
  static constexpr int BUF_COLS = MMA_WARPS * ACC_COLS;      // one accumulator buffer
  static constexpr uint32_t TMEM_COLS = 2 * BUF_COLS;        // double buffered
  static_assert(TMEM_COLS <= 512, "TMEM columns");
  static_assert(MMA_WARPS <= 2, "one drain barrier per MMA issuer (SharedState::drain)");
  static_assert(B_STAGES <= MAX_B_STAGES, "weight ring barriers");
  // The token producer reuses a token stage once the MMAs of the K-block
  // A_STAGES earlier have completed, which it learns from that K-block's
  // weight-stage "empty" barrier; with B_STAGES >= A_STAGES that barrier cannot
  // have moved on by a further phase before the producer looks.
  static_assert(B_STAGES >= A_STAGES, "token stages are released through the weight ring");
  // Each stage must always be consumed by the same issuer (stage s by issuer
  // s % MMA_WARPS): mbarrier waits tell phases apart only modulo 2, so a warp
  // may never skip a use of a stage it waits on.  With both rings multiples of
  // the issuer count and every tile's K-blocks padded to whole rounds, stage
  // and issuer stay paired.
  static_assert(A_STAGES % MMA_WARPS == 0 && B_STAGES % MMA_WARPS == 0,
                "stages pair with issuers");
  static constexpr uint32_t IDESC = ptx::idesc_bf16_f32(BM, MMA_N);
};

struct SharedState {
  uint64_t a_full[A_STAGES];       // token tile landed (TMA transaction bytes)
  uint64_t b_full[MAX_B_STAGES];   // weight tile landed
  uint64_t b_empty[MAX_B_STAGES];  // the K-block's MMAs completed (tcgen05.commit)
  uint64_t tq_full[TILE_Q], tq_empty[TILE_Q];
  int tq_tile[TILE_Q];
  uint64_t tmem_full[2];
  uint64_t tmem_empty[2];
  uint64_t drain[2];
  uint32_t tmem_base;
  int abort;
  int last;        // this CTA took the last exit ticket
  TileMap tm;
};

template <int MMA_N>
__global__ void __launch_bounds__(THREADS, 1) grouped_gemm_kernel(const __grid_constant__ GemmParams p) {
  using Sh = Shape<MMA_N>;
  constexpr int B_STAGES = Sh::B_STAGES;
  constexpr int B_BYTES = Sh::B_BYTES;
  constexpr int ACC_COLS = Sh::ACC_COLS;
  constexpr uint32_t TMEM_COLS = Sh::TMEM_COLS;
  constexpr uint32_t IDESC = Sh::IDESC;
  constexpr int MW = Sh::MMA_WARPS;
  constexpr int BUF_COLS = Sh::BUF_COLS;
  constexpr int HALF = MMA_N / 2;  // gate/up: W1 rows [0, HALF), W3 rows [HALF, MMA_N)
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte aligned operand rings (128-byte swizzle atoms span 1024 bytes):
  // the token ring, then the weight ring
  const uint32_t raw_addr = ptx::smem_addr(smem_raw);
  uint8_t* ring_a = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
  uint8_t* ring_b = ring_a + A_STAGES * A_BYTES;
  SharedState& ss = *reinterpret_cast<SharedState*>(ring_b + B_STAGES * B_BYTES);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  ptx::pdl_launch_dependents();
  if (warp == 1) {
    ptx::tmem_alloc(&ss.tmem_base, TMEM_COLS);
    ptx::tmem_relinquish();
  }
  if (threadIdx.x == 0) {
    for (int i = 0; i < A_STAGES; ++i) ptx::mbar_init(&ss.a_full[i], 1);
    for (int i = 0; i < B_STAGES; ++i) {
      ptx::mbar_init(&ss.b_full[i], 1);
      ptx::mbar_init(&ss.b_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(&ss.tmem_full[i], MW);
      ptx::mbar_init(&ss.tmem_empty[i], 4);
    }
    ptx::mbar_init(&ss.drain[0], 1);
    ptx::mbar_init(&ss.drain[1], 1);
    for (int i = 0; i < TILE_Q; ++i) {
      ptx::mbar_init(&ss.tq_full[i], 1);
      // the token producer, the MMA issuers and the epilogue warps take each tile
      ptx::mbar_init(&ss.tq_empty[i], 1 + MW + EPI_WARPS);
    }
    ss.abort = 0;
    ptx::fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    ptx::tma_prefetch_desc(&p.pr[0].a_r);
  } else if (warp == BPROD_WARP && lane == 0) {
    ptx::tma_prefetch_desc(&p.pr[0].b0_r);
    ptx::tma_prefetch_desc(&p.pr[0].b1_r);
  }
  // everything below reads what earlier kernels in the stream wrote
  ptx::pdl_wait();

  // The weight producer claims the CTA's first tile now: the claim's latency
  // hides under the construction of the tile map.
  int first = 0;
  if (warp == BPROD_WARP && lane == 0) first = first_tile(p);
  // Routed row-tile map from the group offsets.
  if (warp == 2) build_tile_map(ss.tm, p, lane);
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();

  const uint32_t tmem_base = ss.tmem_base;
  const int tiles0 = problem_tiles(p.pr[0], ss.tm, p);
  const int total = tiles0 + (p.nprob > 1 ? problem_tiles(p.pr[1], ss.tm, p) : 0);
  volatile int* abort = &ss.abort;

  if (warp == BPROD_WARP) {
    // ---------------- weight producer and tile claimer ----------------
    if (lane == 0) {
      const uint64_t w_policy = ptx::l2_policy_evict_first();
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued_mask = 0, last_parity = 0;
      int qslot = 0;
      uint32_t qphase = 0;
      int tile = first;
      int next = tile < total ? claim_tile(p, tile) : total;
      for (;;) {
        // hand the tile (or the end mark) to the other roles
        if (!ptx::mbar_wait(&ss.tq_empty[qslot], qphase ^ 1u, abort)) break;
        ss.tq_tile[qslot] = tile < total ? tile : -1;
        ptx::mbar_arrive(&ss.tq_full[qslot]);
        if (++qslot == TILE_Q) { qslot = 0; qphase ^= 1u; }
        if (tile >= total) break;
        const TileInfo ti = decode_tile(tile, ss.tm, p, tiles0);
        const Problem& P = p.pr[ti.prob];
        const CUtensorMap* b0 = ti.shared ? &P.b0_s : &P.b0_r;
        const CUtensorMap* b1 = ti.shared ? &P.b1_s : &P.b1_r;
        const int b_row = ti.grp * (ti.shared ? P.b_s_group_rows : P.b_r_group_rows) + ti.n0;
        int kbeg, K;
        tile_k_range(ti, P, &kbeg, &K);
        const int nk = (K + BK - 1) / BK;
        bool ok = true;
        for (int kb = 0; kb < round_up(nk, MW); ++kb) {
          if (!ptx::mbar_wait(&ss.b_empty[stage], phase ^ 1u, abort)) { ok = false; break; }
          if (kb >= nk) {
            ptx::mbar_arrive(&ss.b_full[stage]);   // padding stage: no data
          } else {
            uint8_t* sb = ring_b + stage * B_BYTES;
            const int xb = kbeg + kb * BK;
            ptx::mbar_arrive_expect_tx(&ss.b_full[stage], B_BYTES);
            if (p.weights_once) {
              // weight tiles read once: evict them first, keeping the activations
              // and expert outputs in L2 for the down tiles and the merge
              ptx::tma_load_2d_hint(sb, b0, &ss.b_full[stage], xb, b_row, w_policy);
              if (P.gateup)
                ptx::tma_load_2d_hint(sb + HALF * BK * 2, b1, &ss.b_full[stage], xb, b_row,
                                      w_policy);
            } else {
              ptx::tma_load_2d(sb, b0, &ss.b_full[stage], xb, b_row);
              if (P.gateup)
                ptx::tma_load_2d(sb + HALF * BK * 2, b1, &ss.b_full[stage], xb, b_row);
            }
          }
          issued_mask |= 1u << stage;
          last_parity = (last_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == B_STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        tile = next;
        next = tile < total ? claim_tile(p, tile) : total;
      }
      // every issued load has landed before the CTA may retire
      for (int s = 0; s < B_STAGES; ++s)
        if (issued_mask & (1u << s)) wait_drain(&ss.b_full[s], (last_parity >> s) & 1u, abort);
    }
  } else if (warp == 0) {
    // ---------------- token / activation producer ----------------
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued_mask = 0, last_parity = 0;
      // position, in the weight ring, of the K-block A_STAGES behind this one
      int rstage = 0;
      uint32_t rphase = 0;
      int lag = A_STAGES;  // K-blocks still to go before that position exists
      int qslot = 0;
      uint32_t qphase = 0;
      for (;;) {
        if (!ptx::mbar_wait(&ss.tq_full[qslot], qphase, abort)) break;
        const int tile = *reinterpret_cast<volatile int*>(&ss.tq_tile[qslot]);
        ptx::mbar_arrive_after_reads(&ss.tq_empty[qslot]);
        if (++qslot == TILE_Q) { qslot = 0; qphase ^= 1u; }
        if (tile < 0) break;
        const TileInfo ti = decode_tile(tile, ss.tm, p, tiles0);
        const Problem& P = p.pr[ti.prob];
        if (ti.prob == 1) {
          // the activations of this group come from problem 0's epilogues
          const int g = ti.shared ? p.E + ti.grp : ti.grp;
          if (!ptx::counter_wait(p.counters + g, rows_ready_target(p, ti), abort)) break;
          ptx::fence_proxy_async_global();
        }
        const CUtensorMap* amap = ti.shared ? &P.a_s : &P.a_r;
        const int a_row = ti.shared                    ? ti.grp * P.a_s_group_stride + ti.m0
                          : (p.dense_a && ti.prob == 0) ? ti.m0
                                                        : ti.row0 + ti.m0;
        int kbeg, K;
        tile_k_range(ti, P, &kbeg, &K);
        const int nk = (K + BK - 1) / BK;
        bool ok = true;
        for (int kb = 0; kb < round_up(nk, MW); ++kb) {
          // the stage's previous K-block (A_STAGES back) has finished its MMAs
          if (lag > 0) {
            --lag;
          } else {
            if (!ptx::mbar_wait(&ss.b_empty[rstage], rphase, abort)) { ok = false; break; }
            if (++rstage == B_STAGES) { rstage = 0; rphase ^= 1u; }
          }
          if (kb >= nk) {
            ptx::mbar_arrive(&ss.a_full[stage]);   // padding stage: no data
          } else {
            uint8_t* sa = ring_a + stage * A_BYTES;
            const int xb = kbeg + kb * BK;
            const int xa = P.a_k_mod > 0 ? xb % P.a_k_mod : xb;
            ptx::mbar_arrive_expect_tx(&ss.a_full[stage], A_BYTES);
            ptx::tma_load_2d(sa, amap, &ss.a_full[stage], xa, a_row);
          }
          issued_mask |= 1u << stage;
          last_parity = (last_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == A_STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
      }
      for (int s = 0; s < A_STAGES; ++s)
        if (issued_mask & (1u << s)) wait_drain(&ss.a_full[s], (last_parity >> s) & 1u, abort);
    }
  } else if (warp == 1 || (MW > 1 && warp == MMA_WARP1)) {
    // ---------------- MMA issuers ----------------
    // Issuer m takes the K-blocks kb with kb % MW == m of every tile into
    // accumulator m of the tile's buffer; all issuers walk the same stages.
    // The whole warp walks the loop, its waits decided by a warp vote, and an
    // elected lane issues each tcgen05 operation (the operands stay
    // warp-uniform, which issues the MMAs about a quarter faster than one lane
    // looping alone).
    const int m = warp == 1 ? 0 : 1;
    int astage = 0, bstage = 0;
    uint32_t aphase = 0, bphase = 0;
    int acc = 0;
    uint32_t acc_phase = 0;
    int qslot = 0;
    uint32_t qphase = 0;
    for (;;) {
      if (!__all_sync(kWarpMask, ptx::mbar_wait(&ss.tq_full[qslot], qphase, abort))) break;
      const int tile = __shfl_sync(kWarpMask, *reinterpret_cast<volatile int*>(&ss.tq_tile[qslot]), 0);
      __threadfence_block();   // the slot is read before the warp hands it back
      __syncwarp();
      ptx::mbar_arrive_elect(&ss.tq_empty[qslot]);
      if (++qslot == TILE_Q) { qslot = 0; qphase ^= 1u; }
      if (tile < 0) break;
      const TileInfo ti = decode_tile(tile, ss.tm, p, tiles0);
      int kbeg, K;
      tile_k_range(ti, p.pr[ti.prob], &kbeg, &K);
      const int nk = (K + BK - 1) / BK;
      if (!__all_sync(kWarpMask, ptx::mbar_wait(&ss.tmem_empty[acc], acc_phase ^ 1u, abort)))
        break;
      ptx::tc_fence_after();
      const uint32_t d_tmem = tmem_base + acc * BUF_COLS + m * ACC_COLS;
      bool ok = true;
      uint32_t accumulate = 0;
      for (int kb = 0; kb < round_up(nk, MW); ++kb) {
        const int ca = astage, cb = bstage;
        const uint32_t pa = aphase, pb = bphase;
        if (++astage == A_STAGES) { astage = 0; aphase ^= 1u; }
        if (++bstage == B_STAGES) { bstage = 0; bphase ^= 1u; }
        if (kb % MW != m) continue;
        const bool ready =
            ptx::mbar_wait(&ss.a_full[ca], pa, abort) && ptx::mbar_wait(&ss.b_full[cb], pb, abort);
        if (!__all_sync(kWarpMask, ready)) {
          ok = false;
          break;
        }
        if (kb < nk) {
          ptx::tc_fence_after();
          // descriptor start-address fields count 16-byte units: +2 per K step
          const uint64_t a_desc = ptx::smem_desc_sw128(ptx::smem_addr(ring_a + ca * A_BYTES));
          const uint64_t b_desc = ptx::smem_desc_sw128(ptx::smem_addr(ring_b + cb * B_BYTES));
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            ptx::mma_f16_ss_elect(d_tmem, a_desc + 2 * kk, b_desc + 2 * kk, IDESC, accumulate);
            accumulate = 1;
          }
        }
        // frees the weight stage, and the token stage to the producer's next
        // lap, when these MMAs finish
        ptx::mma_commit_elect(&ss.b_empty[cb]);
      }
      if (!ok) break;
      ptx::mma_commit_elect(&ss.tmem_full[acc]);   // accumulator ready for the epilogue
      if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
    }
    __syncwarp();
    ptx::mma_commit_elect(&ss.drain[m]);
    wait_drain(&ss.drain[m], 0, abort);
  } else if (warp >= 2 && warp < 6) {
    // ---------------- epilogue (warps 2..5) ----------------
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    int acc = 0;
    uint32_t acc_phase = 0;
    int qslot = 0;
    uint32_t qphase = 0;
    for (;;) {
      if (!ptx::mbar_wait(&ss.tq_full[qslot], qphase, abort)) break;
      const int tile = *reinterpret_cast<volatile int*>(&ss.tq_tile[qslot]);
      __threadfence_block();   // the slot is read before lane 0 hands it back
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&ss.tq_empty[qslot]);
      if (++qslot == TILE_Q) { qslot = 0; qphase ^= 1u; }
      if (tile < 0) break;
      const TileInfo ti = decode_tile(tile, ss.tm, p, tiles0);
      const Problem& P = p.pr[ti.prob];
      int kbeg, K;
      tile_k_range(ti, P, &kbeg, &K);
      const bool two = MW > 1 && K > BK;   // the second accumulator holds K-blocks
      if (!ptx::mbar_wait(&ss.tmem_full[acc], acc_phase, abort)) break;
      ptx::tc_fence_after();
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + acc * BUF_COLS;
      const int r = ti.m0 + q * 32 + lane;   // accumulator row of this lane
      bool row_ok = r < ti.rows;
      size_t out_row = (size_t)ti.row0 + r;
      if (p.dense_a && ti.prob == 0 && !ti.shared) {
        // row r is token r: kept if the token chose this tile's expert
        row_ok = false;
        if (r < p.T) {
          int hit = -1;
          for (int j0 = 0; j0 < p.k; j0 += 8) {
            int ev[8];
#pragma unroll
            for (int u = 0; u < 8; ++u)
              ev[u] = (j0 + u < p.k) ? __ldcg(p.idx + (size_t)r * p.k + j0 + u) : -1;
#pragma unroll
            for (int u = 0; u < 8; ++u)
              if (ev[u] == ti.grp) hit = j0 + u;
          }
          if (hit >= 0) {
            row_ok = true;
            if (p.mask) {
              // the pair's row: the group's offset plus the tokens below r
              // that chose the same expert; column tile 0 records it in inv
              const uint32_t* m = p.mask + (size_t)ti.grp * p.mask_stride;
              const int word = r >> 5;
              int rank = __popc(__ldg(m + word) & ((1u << (r & 31)) - 1u));
              for (int w = 0; w < word; ++w) rank += __popc(__ldg(m + w));
              out_row = (size_t)ss.tm.off[ti.grp] + rank;
              if (ti.n0 == 0) p.inv_out[(size_t)r * p.k + hit] = (int32_t)out_row;
            } else {
              out_row = (size_t)__ldcg(p.inv + (size_t)r * p.k + hit);
            }
          }
        }
      }
      store_tile<MMA_N>(ti, P, taddr, ACC_COLS, two, row_ok, out_row);
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&ss.tmem_empty[acc]);
      if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
      if (p.nprob > 1 && ti.prob == 0) release_rows(p, ti, lane);
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem_base, TMEM_COLS);
  }
  if (threadIdx.x == 0 && ss.abort && p.status) atomicOr(p.status, kStTimeout);
  reset_counters_at_exit_block(p, &ss.last);
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
bool make_map(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows) {
  return make_tensor_map(m, base, rows, cols, box_rows, BK, 2, 128);
}

template <int MMA_N>
constexpr size_t smem_bytes() {
  return 1024 + A_STAGES * A_BYTES + Shape<MMA_N>::B_STAGES * Shape<MMA_N>::B_BYTES +
         sizeof(SharedState);
}
static_assert(smem_bytes<256>() <= 227 * 1024 && smem_bytes<128>() <= 227 * 1024,
              "shared memory budget");

template <int MMA_N>
cudaError_t launch_one(const GemmParams& p, int tiles_upper, cudaStream_t st, int max_ctas = 0) {
  static std::atomic<uint64_t> smem_set{0};
  const cudaError_t e = set_smem_once(grouped_gemm_kernel<MMA_N>, (int)smem_bytes<MMA_N>(), smem_set);
  if (e != cudaSuccess) return e;
  int grid = num_sms();
  if (max_ctas > 0 && max_ctas < grid) grid = max_ctas;
  if (tiles_upper < grid) grid = tiles_upper;
  if (grid < 1) grid = 1;
  return launch_pdl(grouped_gemm_kernel<MMA_N>, dim3(grid), dim3(THREADS), smem_bytes<MMA_N>(),
                    st, p);
}

}  // namespace

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  // looked up once (a function-local static is initialised once, thread-safely)
  static const EncodeTiledFn fn = [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<EncodeTiledFn>(ptr);
    return static_cast<EncodeTiledFn>(nullptr);
  }();
  return fn;
}

bool make_tensor_map(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols,
                     uint32_t box_rows, uint32_t box_cols, int elem_bytes, int swizzle_bytes) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * (cuuint64_t)elem_bytes};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUtensorMapDataType dt = elem_bytes == 4   ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32
                                 : elem_bytes == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                                   : CU_TENSOR_MAP_DATA_TYPE_UINT8;
  return fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE,
            swizzle_bytes == 128  ? CU_TENSOR_MAP_SWIZZLE_128B
            : swizzle_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                  : CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

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
  const bool dense = a.dense_a != 0;
  bool ok = (dense ? make_map(&G.a_r, a.h, a.T, a.D, BM)
                   : make_map(&G.a_r, a.xperm, rows_r, a.D, BM)) &&
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
  p.sched = a.counters + a.E + a.S;   // zeroed with the group counters
  // small batches: about one row tile per expert, so each weight tile is read
  // once (decode: 5 % faster); large batches re-read them from L2
  p.weights_once = narrow ? 1 : 0;
  p.nprob = 2;
  p.E = a.E; p.S = a.S; p.T = a.T;
  p.rows_r = rows_r;
  p.dense_a = dense ? 1 : 0;
  p.k = a.k;
  p.idx = a.idx;
  p.inv = a.inv;
  // one part of the groups: the routed experts (no shared tiles), or the
  // shared experts (no routed groups; their counters live in counters_s)
  int mt_r = mt_upper, S = a.S;
  if (a.part == kFfnRouted) {
    p.S = S = 0;
  } else if (a.part == kFfnShared) {
    p.E = 0;
    mt_r = 0;
    p.counters = a.counters_s;
    p.sched = a.counters_s + a.S;
    p.exit_ticket = a.counters_s + a.S + 1;
    p.nreset = a.S;
  }
  if (a.mask) {
    p.mask = a.mask;
    p.mask_stride = a.mask_stride;
    p.counts_out = a.counts_out;
    p.offsets_out = a.offsets_out;
    p.touched_out = a.touched_out;
    p.inv_out = a.inv_out;
  }
  if (a.self_reset && a.part != kFfnShared) {
    p.exit_ticket = a.counters + a.E + a.S + 1;
    p.nreset = a.E + a.S;
  }
  const int tiles_g = mt_r * ((a.F + half - 1) / half) + S * mt_s * ((a.Fs + half - 1) / half);
  const int nt_d = (a.D + nmma - 1) / nmma;
  const int tiles_d = mt_r * nt_d + S * mt_s * nt_d;
  cudaError_t err = narrow ? launch_one<128>(p, tiles_g + tiles_d, st, a.max_ctas)
                           : launch_one<256>(p, tiles_g + tiles_d, st, a.max_ctas);
  if (err == cudaSuccess && marks) err = cudaEventRecord(static_cast<cudaEvent_t>(marks[0]), st);
  *nlaunch += 1;
  return err;
}

}  // namespace moe
