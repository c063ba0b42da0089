// Grouped expert MLPs with FP8 weights (E4M3 codes, one power-of-two scale per
// 128 x 128 block) and bf16 activations, on the 5th-generation tensor cores.
//
// The layer is the one the bf16 kernel computes -- act = silu(x W1^T) * (x W3^T)
// per routed expert on the rows grouped to it and per shared expert on every
// token, then y = act W2^T ("GLM-5.2", PocketLLM, Implemented execution path;
// "Model anatomy -- GLM-5.2", MoE panel) -- with each weight read as
// e4m3(code) * 2^e.  Decoded weights are exact bf16 values and the
// activations stay bf16, so the products are those of the bf16 path on the
// decoded weights; only the weight stream is halved, which is what a decode
// batch (bound by reading the touched experts' weights) gains from.
//
// The MMA has the weights as its A operand, read from tensor memory, and the
// tokens as its B operand, read from shared memory (D^T = W . X^T):
//   * the FP8 tile goes HBM -> shared memory (TMA) -> registers, is decoded
//     there and written to TMEM with tcgen05.st, so the bf16 copy of the
//     weights never passes through shared memory;
//   * a tile covers the tokens of one group in blocks of up to NT (128 or 256)
//     rows, and the MMA's N is the block's row count rounded up to 16, so a
//     group of 40 tokens costs 48 columns of tensor work, not 128 rows.
// Tiles:
//   gate/up  one group x 64 features x a token block: the 128-row A operand
//            stacks W1 and W3 rows so that TMEM lane quarter q holds gate rows
//            (lanes 0-15) and up rows (lanes 16-31) of the same 16 features,
//            and the epilogue warp pairs them with one lane shuffle;
//   down     one group x 128 output columns x a token block.
// Ordering, dynamic tile claiming (every tile, the first one included, from
// the workspace counter, so waits never depend on CTAs that are not resident)
// and the gate/up -> down hand-off (per-group counters, bounded acquire waits)
// are those of the bf16 kernel.
//
// CTA (512 threads, one per SM):
//   warp 0      token producer: TMA of token tiles (bf16, 128-byte swizzle,
//               boxes of 64 rows); waits for the gate/up -> down hand-off.
//   warp 10     weight producer: TMA of FP8 weight tiles (64-byte swizzle) on
//               a ring of its own (12 stages for NT = 128, 8 for NT = 256),
//               running ahead of the tokens.
//   warp 1      MMA issuer and TMEM allocator (512 columns):
//               tcgen05.mma.cta_group::1.kind::f16, M = 128, N <= NT, K = 16.
//               The weights are bf16 in the MMA, so a stage of 8 KB of codes
//               costs as many MMAs as 16 KB of bf16 weights.  The whole warp
//               walks the issue loop and an elected lane issues (~150 cycles
//               per MMA); one commit per K-block frees both the token and the
//               decoded-weight stage.  (Warp 11 is a second issuer when
//               Cfg::MMA_WARPS = 2: K-blocks alternate between two
//               accumulators that the epilogue adds.)
//   warps 2-5   epilogue (tcgen05.ld of the accumulators, SiLU gate or fp32
//               store).
//   warps 6-9,  decoders, two sets of four taking alternate stages: each
//   12-15       warp reads its 32 weight rows of a stage (one row per thread,
//               64 codes), decodes, and stores them to its TMEM lane quarter.
// TMEM columns: accumulator buffers first (two of 128 for NT = 128, so the
// epilogue of one tile overlaps the MMAs of the next; one of 256 for
// NT = 256), then the decoded-weight stages (32 columns each).
#include <cuda_bf16.h>

#include "ffn_common.cuh"
#include "fp8_convert.cuh"

namespace moe {
namespace {

using namespace ffn;

constexpr int W_ROWS = 128;                      // MMA M: weight rows of a tile
constexpr int GU_FEATS = 64;                     // gate/up tile: 64 W1 + 64 W3 rows
constexpr int TOK_BOX = 64;                      // token rows per TMA box
constexpr int TOK_BOX_BYTES = TOK_BOX * BK * 2;  // 8 KiB
constexpr int W8_BYTES = W_ROWS * BK;            // 8 KiB of codes per stage
constexpr uint32_t A_STAGE_COLS = BK / 2;        // 128 lanes x 64 bf16
constexpr uint32_t TMEM_COLS = 512;
constexpr int TPROD_WARP = 0;                    // token producer
constexpr int MMA_WARP0 = 1;                     // MMA issuer (and TMEM allocator)
constexpr int WPROD_WARP = 10;                   // weight producer
constexpr int MMA_WARP1 = 11;                    // second MMA issuer (Cfg::MMA_WARPS = 2)
constexpr int MAX_MMA_WARPS = 2;
constexpr int DEC_SETS = 2;                      // decoder sets: warps 6-9, 12-15
constexpr int THREADS = 16 * 32;
constexpr int DEC_THREADS = 128;
constexpr int MAX_STAGES = 6;
constexpr int MAX_W8_STAGES = 16;

// Role of a warp: MMA issuer index (or -1) and decoder set (or -1).
__device__ __forceinline__ int mma_index(int warp) {
  return warp == MMA_WARP0 ? 0 : warp == MMA_WARP1 ? 1 : -1;
}
__device__ __forceinline__ int decoder_set(int warp) {
  return (warp >= 6 && warp < 10) ? 0 : (warp >= 12 && warp < 16) ? 1 : -1;
}

// Per-NT configuration.
//   STAGES     depth of the token ring and of the decoded-weight ring in TMEM;
//              the two advance together (one stage per K-block) and share
//              their "empty" barrier, so one tcgen05.commit per K-block
//              releases both.
//   W8_STAGES  depth of the FP8 code ring (HBM latency is the longest).
//   MMA_WARPS  issuing warps; with two, a tile's K-blocks alternate between
//              two accumulators (K-block kb -> D_{kb mod 2}) that the epilogue
//              adds.  One warp issuing with elect.sync is faster than two at
//              decode (FFN 0.161 vs 0.165 ms) and leaves TMEM for a second
//              accumulator buffer.
//   ACC_BUFS   accumulator buffers: two where TMEM holds them next to the
//              weight stages, so a tile's epilogue does not hold up the next
//              tile's MMAs (decode down tiles run only 32 K-blocks).
template <int NT>
struct Cfg {
  static constexpr int TOK_STAGE_BYTES = NT * BK * 2;
  static constexpr int MMA_WARPS = 1;
  static constexpr int STAGES = NT == 128 ? 6 : 4;
  static constexpr int ACC_BUFS =
      2 * MMA_WARPS * NT + STAGES * (int)A_STAGE_COLS <= (int)TMEM_COLS ? 2 : 1;
  static constexpr uint32_t BUF_COLS = MMA_WARPS * NT;    // one accumulator buffer
  static constexpr uint32_t A_COL0 = ACC_BUFS * BUF_COLS; // weight stages follow the accumulators
  static constexpr int W8_STAGES = NT == 128 ? 12 : 8;
  static_assert(STAGES <= MAX_STAGES && W8_STAGES <= MAX_W8_STAGES, "ring sizes");
  static_assert(MMA_WARPS <= MAX_MMA_WARPS, "one drain barrier per MMA issuer");
  // Every stage must always meet the same MMA issuer and the same decoder set:
  // mbarrier waits tell phases apart only modulo 2, so a warp may never skip a
  // use of a stage it waits on.  Ring depths are multiples of the issuer and
  // set counts, and every tile's K-blocks are padded to whole issuer rounds.
  static_assert(STAGES % MMA_WARPS == 0 && STAGES % DEC_SETS == 0, "stages pair with warps");
  static_assert(W8_STAGES % DEC_SETS == 0, "code stages pair with decoder sets");
  static_assert(A_COL0 + STAGES * A_STAGE_COLS <= TMEM_COLS, "weight stages fit in TMEM");
};

struct SharedState8 {
  uint64_t tok_full[MAX_STAGES];      // token tile landed (TMA transaction bytes)
  uint64_t a_full[MAX_STAGES];        // decoded weights stored in TMEM (decoder threads)
  uint64_t stage_empty[MAX_STAGES];   // the K-block's MMAs completed (tcgen05.commit)
  uint64_t w8_full[MAX_W8_STAGES], w8_empty[MAX_W8_STAGES];
  uint64_t tmem_full[2], tmem_empty[2];   // per accumulator buffer
  uint64_t drain[MAX_MMA_WARPS];      // one per MMA issuer: its last MMAs completed
  uint64_t tq_full[TILE_Q], tq_empty[TILE_Q];   // claimed tiles, weight producer -> the rest
  int tq_tile[TILE_Q];
  uint32_t tmem_base;
  int abort;
  TileMap tm;
};

// MMA N of a token block that starts `left` rows before the group's end.
template <int NT>
__device__ __forceinline__ int block_n(int left) {
  const int n = (left + 15) & ~15;
  return n < NT ? n : NT;
}

__device__ __forceinline__ uint16_t bf16_bits(float x) {
  return __bfloat16_as_ushort(__float2bfloat16_rn(x));
}

// 16 accumulator columns of this warp's lane quarter: the sum of the tile's
// `nacc` accumulators (its K-blocks split between the MMA issuers), `stride`
// columns apart, added in issuer order.
__device__ __forceinline__ void load_acc(uint32_t taddr, uint32_t stride, int nacc,
                                         uint32_t (&v)[16]) {
  ptx::tmem_ld_x16(taddr, v);
  ptx::tmem_wait_ld();
  for (int a = 1; a < nacc; ++a) {
    uint32_t u[16];
    ptx::tmem_ld_x16(taddr + a * stride, u);
    ptx::tmem_wait_ld();
#pragma unroll
    for (int j = 0; j < 16; ++j)
      v[j] = __float_as_uint(__uint_as_float(v[j]) + __uint_as_float(u[j]));
  }
}

// Gate/up epilogue of one warp: lane i < 16 holds the gate row of feature
// n0 + 16q + i, lane i + 16 the up row of the same feature; columns are the
// block's tokens.  Per 16 tokens the low lanes finish tokens 0-7 and the high
// lanes tokens 8-15, each taking the missing half from its partner lane.
__device__ __forceinline__ void store_gateup(const TileInfo& ti, const Problem& P, uint32_t taddr,
                                             uint32_t stride, int nacc, int n, int q, int lane) {
  const int Nout = ti.shared ? P.N_s : P.N_r;
  const int f = ti.n0 + q * 16 + (lane & 15);
  const bool hi = lane >= 16;
  const bool f_ok = f < Nout;
  uint16_t* out = static_cast<uint16_t*>(ti.shared ? P.out_s : P.out_r);
#pragma unroll 1
  for (int c = 0; c < n; c += 16) {
    uint32_t v[16];
    load_acc(taddr + c, stride, nacc, v);
    const int t0 = ti.m0 + c + (hi ? 8 : 0);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const uint32_t send = hi ? v[j] : v[8 + j];
      const uint32_t recv = __shfl_xor_sync(0xffffffffu, send, 16);
      const float g = __uint_as_float(hi ? recv : v[j]);
      const float u = __uint_as_float(hi ? v[8 + j] : recv);
      const int t = t0 + j;
      if (f_ok && t < ti.rows) out[(size_t)(ti.row0 + t) * Nout + f] = bf16_bits(silu_times(g, u));
    }
  }
}

// Down epilogue of one warp: lane i holds output column n0 + 32q + i.
__device__ __forceinline__ void store_down(const TileInfo& ti, const Problem& P, uint32_t taddr,
                                           uint32_t stride, int nacc, int n, int q, int lane) {
  const int Nout = ti.shared ? P.N_s : P.N_r;
  const int d = ti.n0 + q * 32 + lane;
  const bool d_ok = d < Nout;
  float* out = static_cast<float*>(ti.shared ? P.out_s : P.out_r);
#pragma unroll 1
  for (int c = 0; c < n; c += 16) {
    uint32_t v[16];
    load_acc(taddr + c, stride, nacc, v);
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const int t = ti.m0 + c + j;
      if (d_ok && t < ti.rows) out[(size_t)(ti.row0 + t) * Nout + d] = __uint_as_float(v[j]);
    }
  }
}

__device__ __forceinline__ int tile_k_blocks(const TileInfo& ti, const Problem& P) {
  const int K = ti.shared ? P.K_s : P.K_r;
  return (K + BK - 1) / BK;
}

template <int NT>
__global__ void __launch_bounds__(THREADS, 1) ffn_fp8_kernel(const __grid_constant__ GemmParams p) {
  using C = Cfg<NT>;
  constexpr int S = C::STAGES;
  constexpr int W8S = C::W8_STAGES;
  constexpr int MW = C::MMA_WARPS;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = ptx::smem_addr(smem_raw);
  uint8_t* tok_ring = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
  uint8_t* w8_ring = tok_ring + S * C::TOK_STAGE_BYTES;
  SharedState8& ss = *reinterpret_cast<SharedState8*>(w8_ring + W8S * W8_BYTES);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  ptx::pdl_launch_dependents();
  if (warp == MMA_WARP0) {
    ptx::tmem_alloc(&ss.tmem_base, TMEM_COLS);
    ptx::tmem_relinquish();
  }
  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) {
      ptx::mbar_init(&ss.tok_full[i], 1);
      ptx::mbar_init(&ss.a_full[i], DEC_THREADS);
      ptx::mbar_init(&ss.stage_empty[i], 1);
    }
    for (int i = 0; i < W8S; ++i) {
      ptx::mbar_init(&ss.w8_full[i], 1);
      ptx::mbar_init(&ss.w8_empty[i], DEC_THREADS);
    }
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(&ss.tmem_full[i], MW);
      ptx::mbar_init(&ss.tmem_empty[i], EPI_WARPS);
    }
    for (int i = 0; i < MAX_MMA_WARPS; ++i) ptx::mbar_init(&ss.drain[i], 1);
    // readers of the tile queue: token producer, MMA issuers, 4 epilogue and
    // 8 decoder warps
    for (int i = 0; i < TILE_Q; ++i) {
      ptx::mbar_init(&ss.tq_full[i], 1);
      ptx::mbar_init(&ss.tq_empty[i], 1 + MW + EPI_WARPS + 4 * DEC_SETS);
    }
    ss.abort = 0;
    ptx::fence_barrier_init();
  }
  if (warp == TPROD_WARP && lane == 0) {
    ptx::tma_prefetch_desc(&p.pr[0].a_r);
    ptx::tma_prefetch_desc(&p.pr[0].b0_r);
    ptx::tma_prefetch_desc(&p.pr[0].b1_r);
  }
  // everything below reads what earlier kernels in the stream wrote
  ptx::pdl_wait();

  // The weight producer claims the CTA's first tile now: the claim's latency
  // hides under the construction of the tile map.
  int first = 0;
  if (warp == WPROD_WARP && lane == 0) first = first_tile(p);
  if (warp == 2) build_tile_map<NT>(ss.tm, p, lane);
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();

  const uint32_t tmem_base = ss.tmem_base;
  const int tiles0 = problem_tiles<NT>(p.pr[0], ss.tm, p);
  const int total = tiles0 + (p.nprob > 1 ? problem_tiles<NT>(p.pr[1], ss.tm, p) : 0);
  volatile int* abort = &ss.abort;
  bool bad_exp = false;

  if (warp == TPROD_WARP) {
    // ---------------- token producer ----------------
    if (lane == 0) {
      int ts = 0;
      uint32_t tph = 0;
      uint32_t issued = 0, par = 0;
      int qslot = 0;
      uint32_t qphase = 0;
      for (;;) {
        if (!ptx::mbar_wait(&ss.tq_full[qslot], qphase, abort)) break;
        const int tile = *reinterpret_cast<volatile int*>(&ss.tq_tile[qslot]);
        ptx::mbar_arrive_after_reads(&ss.tq_empty[qslot]);
        if (++qslot == TILE_Q) { qslot = 0; qphase ^= 1u; }
        if (tile < 0) break;
        const TileInfo ti = decode_tile<NT>(tile, ss.tm, p, tiles0);
        const Problem& P = p.pr[ti.prob];
        if (ti.prob == 1) {
          // the activations of this group come from problem 0's epilogues
          const int g = ti.shared ? p.E + ti.grp : ti.grp;
          if (!ptx::counter_wait(p.counters + g, rows_ready_target(p, ti), abort)) break;
          ptx::fence_proxy_async_global();
        }
        const CUtensorMap* amap = ti.shared ? &P.a_s : &P.a_r;
        const int a_row = ti.shared ? ti.grp * P.a_s_group_stride + ti.m0 : ti.row0 + ti.m0;
        const int nk = tile_k_blocks(ti, P);
        const int nbox = (block_n<NT>(ti.rows - ti.m0) + TOK_BOX - 1) / TOK_BOX;
        bool ok = true;
        for (int kb = 0; kb < round_up(nk, MW); ++kb) {
          if (!ptx::mbar_wait(&ss.stage_empty[ts], tph ^ 1u, abort)) { ok = false; break; }
          if (kb >= nk) {
            ptx::mbar_arrive(&ss.tok_full[ts]);   // padding stage: no data
          } else {
            uint8_t* st = tok_ring + ts * C::TOK_STAGE_BYTES;
            ptx::mbar_arrive_expect_tx(&ss.tok_full[ts], nbox * TOK_BOX_BYTES);
            for (int b = 0; b < nbox; ++b)
              ptx::tma_load_2d(st + b * TOK_BOX_BYTES, amap, &ss.tok_full[ts], kb * BK,
                               a_row + b * TOK_BOX);
          }
          issued |= 1u << ts;
          par = (par & ~(1u << ts)) | (tph << ts);
          if (++ts == S) { ts = 0; tph ^= 1u; }
        }
        if (!ok) break;
      }
      // every issued load has landed before the CTA may retire
      for (int s = 0; s < S; ++s)
        if (issued & (1u << s)) wait_drain(&ss.tok_full[s], (par >> s) & 1u, abort);
    }
  } else if (warp == WPROD_WARP) {
    // ---------------- weight producer ----------------
    // Weights depend on nothing the kernel writes, so this warp runs ahead of
    // the token producer (which may wait on the gate/up -> down hand-off) as
    // far as the code ring allows.  It also claims the CTA's tiles (in
    // increasing order, see claim_tile) and publishes each one to the other
    // warps through the tile queue before loading it.
    if (lane == 0) {
      const uint64_t w_policy = ptx::l2_policy_evict_first();
      int ws = 0;
      uint32_t wph = 0;
      uint32_t issued = 0, par = 0;
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
        const TileInfo ti = decode_tile<NT>(tile, ss.tm, p, tiles0);
        const Problem& P = p.pr[ti.prob];
        const CUtensorMap* w0 = ti.shared ? &P.b0_s : &P.b0_r;
        const CUtensorMap* w1 = ti.shared ? &P.b1_s : &P.b1_r;
        const int w_row = ti.grp * (ti.shared ? P.b_s_group_rows : P.b_r_group_rows) + ti.n0;
        const int nk = tile_k_blocks(ti, P);
        bool ok = true;
        for (int kb = 0; kb < round_up(nk, MW); ++kb) {
          if (!ptx::mbar_wait(&ss.w8_empty[ws], wph ^ 1u, abort)) { ok = false; break; }
          if (kb >= nk) {
            ptx::mbar_arrive(&ss.w8_full[ws]);    // padding stage: no data
          } else {
            uint8_t* sw = w8_ring + ws * W8_BYTES;
            ptx::mbar_arrive_expect_tx(&ss.w8_full[ws], W8_BYTES);
            if (p.weights_once) {
              // codes read once: evict them first, keeping tokens and
              // activations in L2
              ptx::tma_load_2d_hint(sw, w0, &ss.w8_full[ws], kb * BK, w_row, w_policy);
              if (P.gateup)
                ptx::tma_load_2d_hint(sw + W8_BYTES / 2, w1, &ss.w8_full[ws], kb * BK, w_row,
                                      w_policy);
            } else {
              ptx::tma_load_2d(sw, w0, &ss.w8_full[ws], kb * BK, w_row);
              if (P.gateup)
                ptx::tma_load_2d(sw + W8_BYTES / 2, w1, &ss.w8_full[ws], kb * BK, w_row);
            }
          }
          issued |= 1u << ws;
          par = (par & ~(1u << ws)) | (wph << ws);
          if (++ws == W8S) { ws = 0; wph ^= 1u; }
        }
        if (!ok) break;
        tile = next;
        next = tile < total ? claim_tile(p, tile) : total;
      }
      for (int s = 0; s < W8S; ++s)
        if (issued & (1u << s)) wait_drain(&ss.w8_full[s], (par >> s) & 1u, abort);
    }
  } else if (mma_index(warp) >= 0 && mma_index(warp) < MW) {
    // ---------------- MMA issuers ----------------
    // Issuer m takes the K-blocks kb with kb % MW == m of every tile into
    // accumulator D_m; all issuers walk the same stage sequence.  The whole
    // warp walks the loop, its waits decided by a warp vote, and an elected
    // lane issues each tcgen05 operation (warp-uniform operands issue faster).
    const int m = mma_index(warp);
    int st = 0;
    uint32_t sph = 0, acc_phase = 0;
    int acc = 0;
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
      const TileInfo ti = decode_tile<NT>(tile, ss.tm, p, tiles0);
      const Problem& P = p.pr[ti.prob];
      const int nk = tile_k_blocks(ti, P);
      const uint32_t idesc = ptx::idesc_bf16_f32(W_ROWS, block_n<NT>(ti.rows - ti.m0));
      if (!__all_sync(kWarpMask, ptx::mbar_wait(&ss.tmem_empty[acc], acc_phase ^ 1u, abort)))
        break;
      ptx::tc_fence_after();
      const uint32_t d_tmem = tmem_base + acc * C::BUF_COLS + m * NT;
      bool ok = true;
      uint32_t accumulate = 0;
      for (int kb = 0; kb < round_up(nk, MW); ++kb) {
        const int cur = st;
        const uint32_t cur_ph = sph;
        if (++st == S) { st = 0; sph ^= 1u; }
        if (kb % MW != m) continue;
        const bool ready = ptx::mbar_wait(&ss.a_full[cur], cur_ph, abort) &&
                           ptx::mbar_wait(&ss.tok_full[cur], cur_ph, abort);
        if (!__all_sync(kWarpMask, ready)) {
          ok = false;
          break;
        }
        if (kb < nk) {
          ptx::tc_fence_after();
          const uint32_t a_tmem = tmem_base + C::A_COL0 + cur * A_STAGE_COLS;
          // descriptor start-address field counts 16-byte units: +2 per K step
          const uint64_t b_desc =
              ptx::smem_desc_sw128(ptx::smem_addr(tok_ring + cur * C::TOK_STAGE_BYTES));
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            ptx::mma_f16_ts_elect(d_tmem, a_tmem + kk * 8, b_desc + 2 * kk, idesc, accumulate);
            accumulate = 1;
          }
        }
        ptx::mma_commit_elect(&ss.stage_empty[cur]);   // token and weight stage free
      }
      if (!ok) break;
      ptx::mma_commit_elect(&ss.tmem_full[acc]);
      if (++acc == C::ACC_BUFS) { acc = 0; acc_phase ^= 1u; }
    }
    __syncwarp();
    ptx::mma_commit_elect(&ss.drain[m]);
    wait_drain(&ss.drain[m], 0, abort);
  } else if (warp >= 2 && warp < 6) {
    // ---------------- epilogue (warps 2..5) ----------------
    const int q = warp & 3;
    uint32_t acc_phase = 0;
    int acc = 0;
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
      const TileInfo ti = decode_tile<NT>(tile, ss.tm, p, tiles0);
      const Problem& P = p.pr[ti.prob];
      const int n = block_n<NT>(ti.rows - ti.m0);
      const int nacc = min(MW, tile_k_blocks(ti, P));
      if (!ptx::mbar_wait(&ss.tmem_full[acc], acc_phase, abort)) break;
      ptx::tc_fence_after();
      const uint32_t taddr =
          tmem_base + (static_cast<uint32_t>(q * 32) << 16) + acc * C::BUF_COLS;
      if (P.gateup) store_gateup(ti, P, taddr, NT, nacc, n, q, lane);
      else store_down(ti, P, taddr, NT, nacc, n, q, lane);
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&ss.tmem_empty[acc]);
      if (++acc == C::ACC_BUFS) { acc = 0; acc_phase ^= 1u; }
      if (p.nprob > 1 && ti.prob == 0) release_rows(p, ti, lane);
    }
  } else if (decoder_set(warp) >= 0) {
    // ---------------- weight decoders (warps 6..9 and 12..15) ----------------
    // Two sets of four warps take alternate stages; each warp decodes the 32
    // weight rows of its TMEM lane quarter.
    const int q = warp & 3;
    const int set = decoder_set(warp);
    const uint32_t t_lanes = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + C::A_COL0;
    int ws = 0, as = 0, seq = 0;
    uint32_t wph = 0, aph = 0;
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
      const TileInfo ti = decode_tile<NT>(tile, ss.tm, p, tiles0);
      const Problem& P = p.pr[ti.prob];
      const int nk = tile_k_blocks(ti, P);
      // this thread's weight row: gate/up stacks the W1 box (64 rows) and the
      // W3 box; lanes 0-15 of quarter q take W1 rows 16q.., lanes 16-31 the
      // W3 rows of the same features; down takes row 32q + lane of one box
      const bool second = P.gateup && lane >= 16;
      const int r = P.gateup ? q * 16 + (lane & 15) : q * 32 + lane;
      const uint32_t row_off = (second ? W8_BYTES / 2 : 0) + r * BK;
      const uint32_t swz = (r >> 1) & 3;   // 64-byte swizzle: chunk c sits at c ^ swz
      const int8_t* ex = ti.shared ? (second ? P.e1_s : P.e0_s) : (second ? P.e1_r : P.e0_r);
      const int rbn = ti.shared ? P.rb_s : P.rb_r;
      const int kbn = ti.shared ? P.kb_s : P.kb_r;
      const int8_t* ex_row = ex + ((size_t)ti.grp * rbn + ti.n0 / fp8::kBlock) * kbn;
      bool ok = true;
      for (int kb = 0; kb < round_up(nk, MW); ++kb) {
        const int my_ws = ws, my_as = as;
        const uint32_t my_wph = wph, my_aph = aph;
        if (++ws == W8S) { ws = 0; wph ^= 1u; }
        if (++as == S) { as = 0; aph ^= 1u; }
        if (seq++ % DEC_SETS != set) continue;
        if (kb >= nk) {
          // padding stage: pass it through both rings with no data
          if (!ptx::mbar_wait(&ss.w8_full[my_ws], my_wph, abort)) { ok = false; break; }
          ptx::mbar_arrive(&ss.w8_empty[my_ws]);
          if (!ptx::mbar_wait(&ss.stage_empty[my_as], my_aph ^ 1u, abort)) { ok = false; break; }
          ptx::mbar_arrive(&ss.a_full[my_as]);
          continue;
        }
        // the exponent load goes out first; the stage wait hides its latency
        const int e = ex_row[(kb * BK) / fp8::kBlock];
        if (!ptx::mbar_wait(&ss.w8_full[my_ws], my_wph, abort)) { ok = false; break; }
        const uint8_t* rowp = w8_ring + my_ws * W8_BYTES + row_off;
        uint4 c4[4];
#pragma unroll
        for (int c = 0; c < 4; ++c)
          c4[c] = *reinterpret_cast<const uint4*>(rowp + ((c ^ swz) << 4));
        ptx::mbar_arrive_after_reads(&ss.w8_empty[my_ws]);
        bad_exp |= !fp8::exp_ok(e);
        const uint32_t s2 = fp8::scale_pair(e);
        uint32_t w[32];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          fp8::decode4(c4[c].x, s2, w[8 * c + 0], w[8 * c + 1]);
          fp8::decode4(c4[c].y, s2, w[8 * c + 2], w[8 * c + 3]);
          fp8::decode4(c4[c].z, s2, w[8 * c + 4], w[8 * c + 5]);
          fp8::decode4(c4[c].w, s2, w[8 * c + 6], w[8 * c + 7]);
        }
        // the stage's previous K-block has been read by its MMAs
        if (!ptx::mbar_wait(&ss.stage_empty[my_as], my_aph ^ 1u, abort)) { ok = false; break; }
        ptx::tc_fence_after();
        ptx::tmem_st_x32(t_lanes + my_as * A_STAGE_COLS, w);
        ptx::tmem_wait_st();
        ptx::tc_fence_before();
        ptx::mbar_arrive(&ss.a_full[my_as]);
      }
      if (!ok) break;
    }
  }

  if (bad_exp && p.status) atomicOr(p.status, kStBounds);
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == MMA_WARP0) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem_base, TMEM_COLS);
  }
  if (threadIdx.x == 0 && ss.abort && p.status) atomicOr(p.status, kStTimeout);
  if (threadIdx.x == 0) reset_counters_at_exit(p);
}

template <int NT>
constexpr size_t smem_bytes8() {
  return 1024 + Cfg<NT>::STAGES * Cfg<NT>::TOK_STAGE_BYTES + Cfg<NT>::W8_STAGES * W8_BYTES +
         sizeof(SharedState8);
}
static_assert(smem_bytes8<256>() <= 227 * 1024 && smem_bytes8<128>() <= 227 * 1024,
              "shared memory budget");
// more than half the SM's shared memory: never two CTAs (two 512-column TMEM
// allocations) on one SM
static_assert(smem_bytes8<128>() > 114 * 1024, "one CTA per SM");

template <int NT>
cudaError_t launch_one8(const GemmParams& p, int tiles_upper, cudaStream_t st, int max_ctas) {
  static std::atomic<uint64_t> smem_set{0};
  const cudaError_t e = set_smem_once(ffn_fp8_kernel<NT>, (int)smem_bytes8<NT>(), smem_set);
  if (e != cudaSuccess) return e;
  int grid = num_sms();
  if (max_ctas > 0 && max_ctas < grid) grid = max_ctas;
  if (tiles_upper < grid) grid = tiles_upper;
  if (grid < 1) grid = 1;
  return launch_pdl(ffn_fp8_kernel<NT>, dim3(grid), dim3(THREADS), smem_bytes8<NT>(), st, p);
}

int cdiv(int a, int b) { return (a + b - 1) / b; }

}  // namespace

// Batches of at most 128 tokens fit every group in one 128-token block (two
// accumulator buffers); larger batches use 256-token blocks.
cudaError_t launch_expert_ffn_fp8(const FfnArgs& a, const Fp8Weights& w, cudaStream_t st,
                                  int* nlaunch, const char** why, void* const* marks) {
  const bool small = a.T <= 128;
  const int nt = small ? 128 : 256;
  const int rows_r = a.T * a.k;
  const int mt_upper = cdiv(rows_r, nt) + a.E;   // sum over experts of ceil(count / nt)
  const int mt_s = cdiv(a.T, nt);

  GemmParams p{};
  Problem& G = p.pr[0];
  Problem& Dn = p.pr[1];
  bool ok = make_tensor_map(&G.a_r, a.xperm, rows_r, a.D, TOK_BOX, BK, 2, 128) &&
            make_tensor_map(&G.b0_r, w.W1, (uint64_t)a.E * a.F, a.D, GU_FEATS, BK, 1, 64) &&
            make_tensor_map(&G.b1_r, w.W3, (uint64_t)a.E * a.F, a.D, GU_FEATS, BK, 1, 64) &&
            make_tensor_map(&Dn.a_r, a.act_r, rows_r, a.F, TOK_BOX, BK, 2, 128) &&
            make_tensor_map(&Dn.b0_r, w.W2, (uint64_t)a.E * a.D, a.F, W_ROWS, BK, 1, 64);
  if (ok && a.S > 0)
    ok = make_tensor_map(&G.a_s, a.h, a.T, a.D, TOK_BOX, BK, 2, 128) &&
         make_tensor_map(&G.b0_s, w.Ws1, (uint64_t)a.S * a.Fs, a.D, GU_FEATS, BK, 1, 64) &&
         make_tensor_map(&G.b1_s, w.Ws3, (uint64_t)a.S * a.Fs, a.D, GU_FEATS, BK, 1, 64) &&
         make_tensor_map(&Dn.a_s, a.act_s, (uint64_t)a.S * a.T, a.Fs, TOK_BOX, BK, 2, 128) &&
         make_tensor_map(&Dn.b0_s, w.Ws2, (uint64_t)a.S * a.D, a.Fs, W_ROWS, BK, 1, 64);
  if (!ok) {
    *why = "cuTensorMapEncodeTiled failed for an FP8 expert operand";
    return cudaErrorInvalidValue;
  }
  const int rbF = cdiv(a.F, fp8::kBlock), rbFs = cdiv(a.Fs, fp8::kBlock);
  const int rbD = cdiv(a.D, fp8::kBlock);

  G.out_r = a.act_r;
  G.out_s = a.act_s;
  G.K_r = a.D; G.K_s = a.D;
  G.N_r = a.F; G.N_s = a.Fs;
  G.a_s_group_stride = 0;
  G.b_r_group_rows = a.F;
  G.b_s_group_rows = a.Fs;
  G.bn_out = GU_FEATS;
  G.gateup = 1;
  G.e0_r = w.W1e; G.e1_r = w.W3e; G.e0_s = w.Ws1e; G.e1_s = w.Ws3e;
  G.rb_r = rbF; G.kb_r = rbD; G.rb_s = rbFs; G.kb_s = rbD;

  Dn.b1_r = Dn.b0_r;
  Dn.b1_s = Dn.b0_s;
  Dn.out_r = a.y;
  Dn.out_s = a.y + (size_t)rows_r * a.D;
  Dn.K_r = a.F; Dn.K_s = a.Fs;
  Dn.N_r = a.D; Dn.N_s = a.D;
  Dn.a_s_group_stride = a.T;
  Dn.b_r_group_rows = a.D;
  Dn.b_s_group_rows = a.D;
  Dn.bn_out = W_ROWS;
  Dn.gateup = 0;
  Dn.e0_r = Dn.e1_r = w.W2e; Dn.e0_s = Dn.e1_s = w.Ws2e;
  Dn.rb_r = rbD; Dn.kb_r = rbF; Dn.rb_s = rbD; Dn.kb_s = rbFs;

  p.offsets = a.offsets;
  p.status = a.status;
  p.counters = a.counters;
  p.nprob = 2;
  p.E = a.E; p.S = a.S; p.T = a.T;
  p.rows_r = rows_r;
  p.weights_once = small ? 1 : 0;   // one 128-token block per group: codes read once
  p.sched = a.counters + a.E + a.S; // tile claims, zeroed with the group counters
  // one part of the groups, as in the bf16 launcher
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
  const int tiles_g = mt_r * cdiv(a.F, GU_FEATS) + S * mt_s * cdiv(a.Fs, GU_FEATS);
  const int tiles_d = (mt_r + S * mt_s) * cdiv(a.D, W_ROWS);
  cudaError_t err = small ? launch_one8<128>(p, tiles_g + tiles_d, st, a.max_ctas)
                          : launch_one8<256>(p, tiles_g + tiles_d, st, a.max_ctas);
  if (err == cudaSuccess && marks) err = cudaEventRecord(static_cast<cudaEvent_t>(marks[0]), st);
  *nlaunch += 1;
  return err;
}

}  // namespace moe
