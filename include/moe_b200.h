/*
 * moe_b200.h -- C ABI of the B200 (sm_100a) GLM-5.2 Mixture-of-Experts
 * feed-forward layer forward pass.
 *
 * The layer ("Model anatomy -- GLM-5.2", frontier-model-atlas, Decoder
 * microscope, Feed-forward / Mixture of Experts panel): E routed experts of
 * which k are active per token, one (in general S) always-on shared expert,
 * learned routing with sigmoid router scores; an expert-score correction bias
 * takes part in the top-k selection only; the selected scores without the
 * bias are renormalised and multiplied by the routed scaling factor (2.5 for
 * GLM-5.2, 1.0 for GLM-4.5-Air per "GLM-4.5 Full Forward", How it works); the
 * weighted expert outputs are merged with the shared expert's output.
 * Sizes ("GLM-5.2", PocketLLM, Model specification): hidden 6144, 256 routed
 * experts, top-8, expert width 2048, 1 shared expert.  Expert weights are
 * named w1/w3 (input projections) and w2 (output projection) ("GLM-5.2",
 * PocketLLM, Implemented execution path); each expert is read as the gated
 * MLP y = w2 (silu(w1 x) * (w3 x)).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Every pointer argument is a DEVICE pointer unless stated otherwise; the
 *    caller allocates and owns every buffer and the stream.  The library never
 *    allocates device memory: all scratch lives in the caller's workspace.
 *  - Arrays are dense and row-major.  Device pointers must be 16-byte aligned.
 *  - bf16 means IEEE bfloat16 stored as uint16_t bit patterns.
 *  - Calls only enqueue work on `stream` and return at once; results are
 *    ready when the stream reaches them.
 *  - Return value: MOE_OK (0), or a negative moe_status_t when the host-side
 *    checks reject the arguments or a launch fails.  On a negative return
 *    nothing was enqueued by the failing step (earlier steps of a composite
 *    call may have been); moe_last_error() gives a message.
 *  - Conditions only the device can see (a non-finite logit, an expert index
 *    out of range, a repeated expert within a token, inconsistent group
 *    offsets, a bounded wait that ran out) raise bits of a status word kept at
 *    the start of the workspace; moe_get_device_status() reads and clears it.
 *    The caller zeroes the workspace once after allocating it (the library
 *    only ever ORs bits into the word, and the counters it keeps there are
 *    left zero by every call that completes).  Kernels never trap; after such
 *    an error, or a negative return from a composite call whose earlier steps
 *    were enqueued, the outputs are unspecified and the workspace is zeroed
 *    again before its next use.
 *  - Limits: 1 <= E <= 1024, 1 <= k <= min(E, 32), 0 <= S <= 16,
 *    T >= 0 (T = 0 enqueues nothing), D, F and Fs positive multiples of 8,
 *    scale finite, T * k < 2^31, and every buffer smaller than 2^31 rows.
 */
#ifndef MOE_B200_H_
#define MOE_B200_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ABI-compatible with cudaStream_t (a pointer to the opaque CUstream_st). */
struct CUstream_st;
typedef struct CUstream_st* moe_stream_t;

/* Layer dimensions. */
typedef struct moe_dims {
  int32_t T;     /* tokens in the batch                                      */
  int32_t D;     /* hidden size                                              */
  int32_t E;     /* routed experts                                           */
  int32_t F;     /* routed expert width (intermediate size)                  */
  int32_t k;     /* experts selected per token                               */
  int32_t S;     /* shared (always-on) experts, 0 allowed                    */
  int32_t Fs;    /* shared expert width                                      */
  float scale;   /* routed scaling factor                                    */
} moe_dims_t;

typedef enum moe_status {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = -1,  /* bad dimension, null or misaligned pointer    */
  MOE_ERR_UNSUPPORTED = -2,  /* no sm_100 device / shape outside the limits  */
  MOE_ERR_CUDA = -3,         /* a CUDA runtime call or launch failed         */
  MOE_ERR_WORKSPACE = -4,    /* workspace missing or smaller than required   */
  MOE_ERR_NONFINITE = -5,    /* device: a router logit was NaN or infinite   */
  MOE_ERR_TIMEOUT = -6,      /* device: a bounded wait gave up               */
  MOE_ERR_BOUNDS = -7        /* device: index/offset out of range or repeated */
} moe_status_t;

/* Bytes of workspace that moe_forward needs for `dims` (a superset of what
 * every other entry point needs).  The workspace must be 256-byte aligned.
 * Returns 0 if the dimensions are invalid. */
size_t moe_workspace_size(const moe_dims_t* dims);

/* Router logits ("Routing: learned", MoE panel; fp32 router):
 *   logits[t, e] = sum_d h[t, d] * Wr[e, d]
 * h [T, D] bf16, Wr [E, D] fp32, logits [T, E] fp32 (output).  fp32-accurate:
 * when D % 64 == 0 and E % 8 == 0 the products run on the tensor cores
 * against an exact three-piece bf16 split of Wr (hi + mid + lo, within 2^-24
 * relative of Wr) with fp32 accumulation; otherwise with fp32 FMAs.  For
 * T <= 256 with E % 64 == 0 one kernel reads Wr itself and splits each tile
 * in shared memory; otherwise the split is written to `ws` first.  Either
 * way the summation order is fixed, so repeated calls give identical bits.
 * `ws` (>= moe_workspace_size bytes) holds the split weight (when written),
 * the partial sums and the status word; it may be NULL only in the small FMA
 * cases that need none of them (then no status is kept). */
int moe_router_logits(const void* h, const float* Wr, const moe_dims_t* dims, float* logits,
                      void* ws, size_t ws_bytes, moe_stream_t stream);

/* Routing (MoE panel: sigmoid scores, bias for selection only, un-biased
 * renormalised scores times the routed scale), one warp per token:
 *   s[e]   = fp32(1 / (1 + exp(-(double)logits[t, e])))
 *   key[e] = s[e] + bias[e]                                   (fp32 add)
 *   idx[t, 0..k-1] = the k experts first under (key descending, index
 *                    ascending), in that order
 *   sum    = s[idx0] + s[idx1] + ... (fp32, slot order)
 *   w[t, j] = (s[idx_j] / sum) * scale                        (fp32 ops)
 * logits [T, E] fp32, bias [E] fp32 -> idx [T, k] int32, w [T, k] fp32.
 * A non-finite logit raises MOE_ERR_NONFINITE in the status word of `ws`
 * (ws may be NULL: then no status is kept). */
int moe_route(const float* logits, const float* bias, const moe_dims_t* dims, int32_t* idx,
              float* w, void* ws, moe_stream_t stream);

/* Group-limited routing ("GLM-4.5 Full Forward", How it works: sigmoid group
 * routing; the pages give neither the rule nor the group counts, so both
 * are parameters and the rule is the reading documented here).  The E
 * experts form n_group contiguous groups of E / n_group.  A group's score is
 * the fp32 sum of its two largest selection keys (its one key for one-expert
 * groups); the topk_group groups first under (score descending, group index
 * ascending) are kept; then idx and w are exactly those of moe_route with
 * the other experts' keys set to -infinity.  n_group = 1 or topk_group =
 * n_group gives moe_route's result.  Limits: 1 <= n_group <= 32, n_group
 * divides E, 1 <= topk_group <= n_group, k <= topk_group * E / n_group.
 * Arguments, layout and errors as moe_route. */
int moe_route_grouped(const float* logits, const float* bias, const moe_dims_t* dims, int n_group,
                      int topk_group, int32_t* idx, float* w, void* ws, moe_stream_t stream);

/* Grouping of the (token, slot) pairs by expert (counting sort; the pages
 * call the expert kernels "grouped"):
 *   counts[e]  = number of pairs routed to expert e            [E] int32
 *   offsets[e] = counts[0] + ... + counts[e-1]                 [E+1] int32
 *   perm[r]    = token of grouped row r; rows offsets[e] .. offsets[e+1]-1
 *                hold expert e's tokens in increasing (token, slot) order
 *                                                              [T*k] int32
 *   inv[t, j]  = grouped row of pair (t, j)                    [T, k] int32
 * idx [T, k] int32 must hold k distinct experts in [0, E) per row; a value
 * out of range or repeated raises MOE_ERR_BOUNDS.  Integer results are
 * exact and deterministic. */
int moe_permute(const int32_t* idx, const moe_dims_t* dims, int32_t* counts, int32_t* offsets,
                int32_t* perm, int32_t* inv, void* ws, size_t ws_bytes, moe_stream_t stream);

/* moe_permute for callers that cannot allocate device memory: the same
 * grouping, bit for bit, with its scratch in a fixed array inside the library
 * instead of a caller workspace.  There is no counterpart on the pages; it
 * exists for callers that must not call cudaMalloc, for example code that
 * runs while another component owns all device memory through a fixed pool,
 * or a serving loop that may not take the device-wide synchronisation an
 * allocation implies, and that therefore cannot provide a workspace.
 *  - Limits: T <= 16384 (64 counting blocks of 256 tokens) and E <= 1024;
 *    larger sizes return MOE_ERR_UNSUPPORTED and enqueue nothing.  The
 *    array (256 KiB) is held by every GPU that loads the library until the
 *    process exits.
 *  - Allocates nothing: no cudaMalloc, cudaFree or allocating library call.
 *  - The first call on each device looks up the array's device address
 *    (cudaGetSymbolAddress) with that device current; make that first call
 *    before any stream capture.
 *  - Every call shares the one array and leaves the last call's contents in
 *    it; each call overwrites every entry it reads, so nothing needs
 *    clearing.  Calls whose work overlaps on the GPU (different streams, or
 *    different host threads) race on the array and give wrong groupings.
 *  - Device-detected errors (an expert index out of range or repeated) are
 *    not recorded: there is no workspace to hold a status word.  With such
 *    an idx, perm and inv are undefined (rows of the offending tokens keep
 *    whatever the buffers held), so validate idx first when it may be bad.
 *  - The looked-up address is cached per device and is not refreshed after
 *    cudaDeviceReset; do not use the library across a device reset. */
int moe_permute_noalloc(const int32_t* idx, const moe_dims_t* dims, int32_t* counts,
                        int32_t* offsets, int32_t* perm, int32_t* inv, moe_stream_t stream);

/* Expert MLPs on grouped rows (gated MLP with w1/w3 -> SiLU gate -> w2):
 *   routed row r (expert e, offsets[e] <= r < offsets[e+1], token perm[r]):
 *     y[r] = W2[e] (silu(W1[e] h[perm[r]]) * (W3[e] h[perm[r]]))
 *   shared row T*k + s*T + t:
 *     y[T*k + s*T + t] = Ws2[s] (silu(Ws1[s] h[t]) * (Ws3[s] h[t]))
 * h [T, D] bf16; perm [T*k], offsets [E+1] int32 as moe_permute writes them;
 * W1, W3 [E, F, D], W2 [E, D, F], Ws1, Ws3 [S, Fs, D], Ws2 [S, D, Fs] bf16
 * (nn.Linear layout: out-features x in-features).  y [T*k + S*T, D] fp32
 * (output).  bf16 tensor-core products with fp32 accumulation; the gated
 * activation is rounded to bf16 before the w2 product.  Ws* may be NULL when
 * S = 0. */
int moe_expert_ffn(const void* h, const int32_t* perm, const int32_t* offsets, const void* W1,
                   const void* W3, const void* W2, const void* Ws1, const void* Ws3,
                   const void* Ws2, const moe_dims_t* dims, float* y, void* ws, size_t ws_bytes,
                   moe_stream_t stream);

/* Merge (MoE panel: weighted expert outputs merged with the always-on shared
 * expert; "Expert fan-out 8 + 1"), deterministic fixed order:
 *   out[t] = sum_s y[T*k + s*T + t] + sum_j w[t, j] * y[inv[t, j]]
 * (fp32: shared experts first, then slots 0..k-1, one fused multiply-add
 * each).  y [T*k + S*T, D] fp32, w [T, k] fp32, inv [T, k] int32 ->
 * out [T, D] fp32.  An inv entry outside [0, T*k) raises MOE_ERR_BOUNDS
 * (ws may be NULL). */
int moe_combine(const float* y, const float* w, const int32_t* inv, const moe_dims_t* dims,
                float* out, void* ws, moe_stream_t stream);

/* The whole layer: moe_router_logits, moe_route, moe_permute, the row
 * gather, moe_expert_ffn and moe_combine in one call on `stream`, with no
 * host synchronisation (capturable in a CUDA graph).  For small batches the
 * shared experts' FFN runs on an internal stream forked from and joined back
 * into `stream` (moe_forward_shared_overlap says when).
 * h [T, D] bf16; Wr [E, D] fp32; bias [E] fp32; weights as in
 * moe_expert_ffn; out [T, D] fp32.  idx_out [T, k] int32 and w_out [T, k]
 * fp32 are optional (NULL: kept in the workspace).  ws_bytes must be at
 * least moe_workspace_size(dims). */
int moe_forward(const void* h, const float* Wr, const float* bias, const void* W1,
                const void* W3, const void* W2, const void* Ws1, const void* Ws3,
                const void* Ws2, const moe_dims_t* dims, float* out, int32_t* idx_out,
                float* w_out, void* ws, size_t ws_bytes, moe_stream_t stream);

/* 1 if moe_forward (bf16 weights, fp8_weights = 0) or moe_forward_fp8
 * (fp8_weights = 1) runs the shared experts' FFN for these dims on an
 * internal stream, next to the routing: the shared experts need no routing,
 * so their weights stream on 32 SMs while the routing kernels run, and the
 * routed experts' FFN launch that follows on `stream` no longer carries them.
 * That is done for bf16 weights when S > 0, T <= 512 and the shared experts'
 * weights are at least 16 MiB (smaller ones cost less than the fork and join
 * save; the FP8 kernel is bound by per-SM MMA issue and decoding, so 32 SMs
 * would finish its shared experts after the routing).  The internal stream
 * and its two events are created on the first such call of each host thread
 * and device and kept for the life of the process; the call still returns
 * without host synchronisation and stays capturable in a CUDA graph (the
 * internal stream forks from and joins back into `stream`).  0 otherwise, or
 * for invalid dims. */
int moe_forward_shared_overlap(const moe_dims_t* dims, int fp8_weights);

/* ---- FP8 expert weights ------------------------------------------------
 * The "Inside GLM" course outline names BF16 and FP8 GLM-5.2 artifacts (its
 * outcomes list and the Release anatomy lesson) but gives no FP8 layout;
 * this library's is: each expert matrix [rows, K] is stored as
 * OCP E4M3 (float8_e4m3fn) codes [rows, K] plus one int8 exponent e per
 * 128 x 128 block ([ceil(rows/128), ceil(K/128)], ragged at the edges), and
 * stands for the weights  w = e4m3(code) * 2^e.  Every such w is exactly a
 * bf16 value for e in [-117, 7]; exponents outside that range, and the NaN
 * codes 0x7F / 0xFF, are outside the format (an exponent outside the range
 * raises MOE_ERR_BOUNDS in the workspace status word; NaN codes are not
 * detected).  Activations stay bf16: the FP8 layer computes exactly what the
 * bf16 layer computes on the decoded weights, with half the weight bytes.
 *
 * Code pointers must be 16-byte aligned; exponent pointers have no
 * alignment rule.  Ws* members may be NULL when S = 0.  The pointed-to
 * arrays are read only, and owned by the caller. */
typedef struct moe_fp8_weights {
  const void* W1;   /* [E, F, D] E4M3 codes */
  const void* W3;   /* [E, F, D] */
  const void* W2;   /* [E, D, F] */
  const void* Ws1;  /* [S, Fs, D] */
  const void* Ws3;  /* [S, Fs, D] */
  const void* Ws2;  /* [S, D, Fs] */
  const int8_t* W1e;   /* [E, ceil(F/128), ceil(D/128)] block exponents */
  const int8_t* W3e;   /* [E, ceil(F/128), ceil(D/128)] */
  const int8_t* W2e;   /* [E, ceil(D/128), ceil(F/128)] */
  const int8_t* Ws1e;  /* [S, ceil(Fs/128), ceil(D/128)] */
  const int8_t* Ws3e;  /* [S, ceil(Fs/128), ceil(D/128)] */
  const int8_t* Ws2e;  /* [S, ceil(D/128), ceil(Fs/128)] */
} moe_fp8_weights_t;

/* moe_expert_ffn with FP8 expert weights (`w8`, device arrays as described
 * above).  Same rows, outputs, workspace and errors as moe_expert_ffn; in
 * addition D, F and Fs (when S > 0) must be multiples of 16 (MOE_ERR_INVALID_ARG
 * otherwise). */
int moe_expert_ffn_fp8(const void* h, const int32_t* perm, const int32_t* offsets,
                       const moe_fp8_weights_t* w8, const moe_dims_t* dims, float* y, void* ws,
                       size_t ws_bytes, moe_stream_t stream);

/* moe_forward with FP8 expert weights: the same pipeline and outputs, with
 * moe_expert_ffn_fp8 in place of moe_expert_ffn (router weight Wr stays
 * fp32).  Same argument rules as moe_forward plus those of
 * moe_expert_ffn_fp8. */
int moe_forward_fp8(const void* h, const float* Wr, const float* bias, const moe_fp8_weights_t* w8,
                    const moe_dims_t* dims, float* out, int32_t* idx_out, float* w_out, void* ws,
                    size_t ws_bytes, moe_stream_t stream);

/* Decodes FP8 weights to bf16 with the same exact decoding the FP8 layer
 * uses: codes [G, R, K] (16-byte aligned), exps [G, ceil(R/128), ceil(K/128)]
 * -> out [G, R, K] bf16 (16-byte aligned), out[g, r, c] = e4m3(code) *
 * 2^exps[g, r/128, c/128].  K must be a multiple of 16.  An exponent outside
 * [-117, 7] raises MOE_ERR_BOUNDS in the status word of `ws` (ws may be
 * NULL: then it is not reported).  G, R, K >= 0; nothing is launched when
 * one is 0. */
int moe_fp8_dequantize(const void* codes, const int8_t* exps, int G, int R, int K, void* out,
                       void* ws, moe_stream_t stream);

/* Row gather, the data movement around the expert-parallel exchange (each
 * rank owns a block of experts; the pages' default multi-GPU layout is expert
 * parallelism, "GLM-5.2" PocketLLM, Implemented execution path):
 *   dst[i] = src[idx[i]],  i < n,
 * rows of row_bytes bytes (a positive multiple of 16), src [src_rows, row_bytes]
 * and dst [n, row_bytes] device buffers (16-byte aligned), idx [n] int32.  An
 * index outside [0, src_rows) zero-fills its row and raises MOE_ERR_BOUNDS in
 * the status word of ws (ws may be NULL: then it is not reported). */
int moe_gather_rows(const void* src, int src_rows, const int32_t* idx, int n, int row_bytes,
                    void* dst, void* ws, moe_stream_t stream);

/* ---- Host-buffer pipeline ----------------------------------------------
 * The layer forward from page-locked host memory to page-locked host memory,
 * for callers whose hidden states live on the host.  The pages' decode
 * profile names host-to-GPU staging (of the active experts) as one of the two
 * hard floors of their runtime ("GLM-5.2" PocketLLM, Validated performance);
 * here the weights stay resident and only the activations cross, overlapped
 * with the layer.  Each submitted step copies h [T, D] bf16 from the host,
 * runs moe_forward / moe_forward_fp8 on the pipeline's compute stream and
 * copies out [T, D] fp32 back to the host.  The input copy runs on one copy
 * stream and the output copy on another, so the copies of step n+1 and n-1
 * overlap the layer of step n; layers run one after another, in submission
 * order, on the compute stream.
 *
 * Memory: the caller owns every buffer.  `dev` (device memory, 256-byte
 * aligned, at least moe_pipeline_device_bytes(dims) bytes) holds two input
 * slots, two output slots and the layer's workspace; it, the weights, Wr
 * and bias must stay valid until moe_pipeline_destroy returns.  The pipeline
 * itself creates two CUDA streams and six events on the current device (no
 * device memory) and frees them in moe_pipeline_destroy.  One pipeline is
 * driven from one host thread at a time. */
typedef struct moe_pipeline moe_pipeline_t;

/* Device bytes a pipeline needs for these dims (0 if the dims are invalid). */
size_t moe_pipeline_device_bytes(const moe_dims_t* dims);

/* Creates a pipeline on the current device.  Weights: bf16 (W1..Ws2 as in
 * moe_forward, w8 = NULL) or FP8 (w8 as in moe_forward_fp8; W1..Ws2 are then
 * ignored and may be NULL).  `stream` is the compute stream (it may be the
 * default stream).  *out receives the handle; on failure *out is NULL and
 * nothing stays allocated. */
int moe_pipeline_create(const moe_dims_t* dims, const float* Wr, const float* bias,
                        const void* W1, const void* W3, const void* W2, const void* Ws1,
                        const void* Ws3, const void* Ws2, const moe_fp8_weights_t* w8,
                        void* dev, size_t dev_bytes, moe_stream_t stream, moe_pipeline_t** out);

/* Enqueues one step: h_host [T, D] bf16 -> out_host [T, D] fp32, both
 * page-locked host memory (cudaHostAlloc / cudaHostRegister; pageable memory
 * is refused with MOE_ERR_INVALID_ARG, since copies from it cannot overlap;
 * with T = 0 nothing is enqueued and the pointers are not looked at).
 * Returns without waiting; h_host must not be modified, and out_host not read,
 * until moe_pipeline_wait returns. */
int moe_pipeline_submit(moe_pipeline_t* p, const void* h_host, float* out_host);

/* Blocks until every submitted step's output is in host memory; returns
 * MOE_OK or the first device-side error of those steps (as
 * moe_get_device_status). */
int moe_pipeline_wait(moe_pipeline_t* p);

/* Waits for outstanding steps, then frees the pipeline's streams and events.
 * NULL is allowed. */
int moe_pipeline_destroy(moe_pipeline_t* p);

/* Routing statistics of the last moe_forward (or moe_permute) that used
 * `ws` with these dims: device pointers into the workspace, valid once the
 * stream has reached the end of that call and until the next call reuses the
 * workspace (the "Inside GLM" course outline's Sparse execution lesson names
 * routed-expert utilisation as a quantity to inspect).
 *   moe_ws_expert_counts   -> int32 [E]: pairs routed to each expert (the
 *                             per-expert load histogram)
 *   moe_ws_touched_experts -> int32 [1]: experts with at least one pair
 * Pointer arithmetic only (no launch, no synchronisation); NULL if ws is NULL
 * or the dims are invalid. */
const int32_t* moe_ws_expert_counts(const void* ws, const moe_dims_t* dims);
const int32_t* moe_ws_touched_experts(const void* ws, const moe_dims_t* dims);

/* Self-test of the bounded device waits (failure detection without a fault):
 * one kernel waits on an mbarrier that nothing arrives on and on a counter
 * that nothing increments, using the same bounded-wait code as the layer's
 * kernels; each wait gives up after about one second.  It records
 * MOE_ERR_TIMEOUT in the status word at the start of `ws` (read it with
 * moe_get_device_status) and returns; the CUDA context stays usable.  Takes
 * about two seconds of GPU time.  `ws` needs at least 256 bytes. */
int moe_selftest_bounded_wait(void* ws, moe_stream_t stream);

/* Self-test of forward progress under shared SMs: launches `nctas` CTAs on
 * `stream`, each holding one SM (120 KB of shared memory, so no expert-FFN CTA
 * fits beside it) for `cycles` SM clock cycles and then returning; they wait
 * on nothing but their own clock.  A layer call issued meanwhile on another
 * stream runs on the SMs that are left, and must finish there: the expert
 * FFN's tiles are claimed only by CTAs that are already running, so none of
 * its waits depends on a CTA that is not resident.
 * nctas in [1, number of SMs], cycles in [0, 2^33] (about 4.4 s at the
 * B200's maximum clock); MOE_ERR_INVALID_ARG otherwise.  No workspace. */
int moe_selftest_occupy(int nctas, long long cycles, moe_stream_t stream);

/* Synchronises `stream`, returns the first error recorded in the status word
 * of `ws` (MOE_OK if none) and clears the word. */
int moe_get_device_status(void* ws, moe_stream_t stream);

/* Message of the last failing call on this host thread ("" if none). */
const char* moe_last_error(void);

/* Number of kernels the last successful call on this host thread enqueued. */
int moe_last_launch_count(void);

/* Stage timing of moe_forward (host-thread local).  `events` points to n
 * cudaEvent_t handles created by the caller; while set, every moe_forward
 * call on this thread records them on its stream at the stage boundaries:
 *   events[0] before the router, [1] after the router logits, [2] after the
 *   routing, [3] after the grouping, [4] after the row gather, [5] after the
 *   expert FFN (gate/up and down GEMMs, one kernel), [6] after the merge.
 * Recording events between the kernels costs their overlapped launches, so
 * profiled steps run a little slower than unprofiled ones.
 * n must be MOE_PROFILE_EVENTS (7) to enable, or 0 (events may be NULL) to
 * disable.  The library keeps the pointer, not a copy: the array must stay
 * valid while enabled. */
#define MOE_PROFILE_EVENTS 7
int moe_set_profile_events(void* const* events, int n);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H_ */
