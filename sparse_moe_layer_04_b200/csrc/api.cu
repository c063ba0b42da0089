// C ABI of the library: argument checks, workspace layout, launches.
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <new>
#include <string>

#include "moe_internal.cuh"

namespace moe {
namespace {

thread_local std::string g_err;
thread_local int g_launches = 0;
thread_local void* const* g_prof_events = nullptr;

// Records stage-boundary event i of moe_forward when profiling is enabled.
cudaError_t mark(int i, cudaStream_t st) {
  if (!g_prof_events) return cudaSuccess;
  return cudaEventRecord(static_cast<cudaEvent_t>(g_prof_events[i]), st);
}

int fail(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_err = buf;
  return code;
}

int cuda_fail(cudaError_t e, const char* what) {
  return fail(MOE_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

constexpr int kMaxDev = 64;
// Longest hold of moe_selftest_occupy: 2^33 cycles, about 4.4 s at 1.965 GHz.
constexpr long long kOccupyMaxCycles = 1ll << 33;

int check_device() {
  static int checked[kMaxDev] = {0};  // 0 unknown, 1 ok, -1 unsupported
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDev) return fail(MOE_ERR_UNSUPPORTED, "device index %d", dev);
  if (checked[dev] == 0) {
    int major = 0, minor = 0;
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
    checked[dev] = (major == 10 && minor == 0) ? 1 : -1;
  }
  if (checked[dev] < 0)
    return fail(MOE_ERR_UNSUPPORTED, "this library is built for sm_100a (B200) devices only");
  return MOE_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_dims(const moe_dims_t* d) {
  if (!d) return fail(MOE_ERR_INVALID_ARG, "dims is NULL");
  if (d->T < 0) return fail(MOE_ERR_INVALID_ARG, "T = %d < 0", d->T);
  if (d->E < 1 || d->E > 1024) return fail(MOE_ERR_INVALID_ARG, "E = %d outside [1, 1024]", d->E);
  if (d->k < 1 || d->k > 32 || d->k > d->E)
    return fail(MOE_ERR_INVALID_ARG, "k = %d outside [1, min(E, 32)]", d->k);
  if (d->D < 8 || d->D % 8) return fail(MOE_ERR_INVALID_ARG, "D = %d not a positive multiple of 8", d->D);
  if (d->F < 8 || d->F % 8) return fail(MOE_ERR_INVALID_ARG, "F = %d not a positive multiple of 8", d->F);
  if (d->S < 0 || d->S > 16) return fail(MOE_ERR_INVALID_ARG, "S = %d outside [0, 16]", d->S);
  if (d->S > 0 && (d->Fs < 8 || d->Fs % 8))
    return fail(MOE_ERR_INVALID_ARG, "Fs = %d not a positive multiple of 8", d->Fs);
  if (!(d->scale == d->scale) || d->scale > 3.4e38f || d->scale < -3.4e38f)
    return fail(MOE_ERR_INVALID_ARG, "scale is not finite");
  const long long rows = (long long)d->T * d->k + (long long)d->S * d->T;
  if (rows >= (1ll << 31)) return fail(MOE_ERR_UNSUPPORTED, "T*k + S*T >= 2^31");
  if ((long long)d->E * d->F >= (1ll << 31) || (long long)d->E * d->D >= (1ll << 31))
    return fail(MOE_ERR_UNSUPPORTED, "E*F or E*D >= 2^31");
  return MOE_OK;
}

#define MOE_CHECK_PTR(p)                                                          \
  do {                                                                            \
    if (!(p)) return fail(MOE_ERR_INVALID_ARG, "%s is NULL", #p);                 \
    if (!aligned16(p)) return fail(MOE_ERR_INVALID_ARG, "%s is not 16-byte aligned", #p); \
  } while (0)

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

struct Ws {
  WsLayout L;
  uint8_t* base;
  template <typename T>
  T* at(size_t off) const { return reinterpret_cast<T*>(base + off); }
  int* status() const { return base ? reinterpret_cast<int*>(base + L.status) : nullptr; }
};

int check_ws(const moe_dims_t* d, void* ws, size_t ws_bytes, Ws* out) {
  if (!ws_layout(*d, &out->L)) return fail(MOE_ERR_INVALID_ARG, "workspace layout overflow");
  if (!ws) return fail(MOE_ERR_WORKSPACE, "workspace is NULL");
  if (reinterpret_cast<uintptr_t>(ws) & 255u)
    return fail(MOE_ERR_WORKSPACE, "workspace is not 256-byte aligned");
  if (ws_bytes < out->L.total)
    return fail(MOE_ERR_WORKSPACE, "workspace has %zu bytes, needs %zu", ws_bytes, out->L.total);
  out->base = static_cast<uint8_t*>(ws);
  return MOE_OK;
}

// Host-side checks come first and touch no CUDA API, so argument errors are
// reported the same way with or without a device.
int begin(const moe_dims_t* d) {
  g_err.clear();
  g_launches = 0;
  return check_dims(d);
}

// Router logits into `dst` (nsplit partial planes, or the logits themselves
// when nsplit == 1).
cudaError_t launch_router(const uint16_t* h, const float* Wr, const moe_dims_t& d,
                          const RouterSplit& sp, const Ws& w, float* dst, cudaStream_t st, int* n,
                          const char** why) {
  if (sp.fused) {
    *n += 1;
    *why = "router launch";
    return launch_router_tc_fused(h, Wr, d.T, d.D, d.E, sp.nsplit, sp.chunk / 64, dst,
                                  w.status(), st, why);
  }
  if (sp.tensor) {
    uint16_t* wr3 = w.at<uint16_t>(w.L.wr3);
    cudaError_t e = launch_split_router(Wr, d.E, d.D, wr3, st);
    if (e != cudaSuccess) {
      *why = "router weight split launch";
      return e;
    }
    e = launch_router_tc(h, wr3, d.T, d.D, d.E, sp.nsplit, sp.chunk, dst, st, why);
    *n += 2;
    return e;
  }
  *why = "router logits launch";
  *n += 1;
  return launch_router_partials(h, Wr, d.T, d.D, d.E, sp, dst, st);
}

}  // namespace

int num_sms() {
  // per-device cache; threads racing on the first call store the same value
  static std::atomic<int> cache[kMaxDev];
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= kMaxDev) return 148;
  int n = cache[dev].load(std::memory_order_relaxed);
  if (!n) {
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
    cache[dev].store(n, std::memory_order_relaxed);
  }
  return n;
}

bool ws_layout(const moe_dims_t& d, WsLayout* L) {
  const size_t T = d.T, D = d.D, E = d.E, F = d.F, k = d.k, S = d.S, Fs = d.S > 0 ? d.Fs : 0;
  const RouterSplit sp = router_split(d.T, d.D, d.E);
  const size_t nblk = (T + kPermBlockTokens - 1) / kPermBlockTokens;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = align256(off + bytes);
    return at;
  };
  L->status = take(256);
  L->ticket = take(256);
  L->partials = take((size_t)sp.nsplit * T * E * 4);
  L->wr3 = take(sp.tensor && !sp.fused ? E * 3 * D * 2 : 0);
  L->idx = take(T * k * 4);
  L->w = take(T * k * 4);
  L->counts = take(E * 4);
  L->offsets = take((E + 1) * 4);
  L->perm = take(T * k * 4);
  L->inv = take(T * k * 4);
  L->blk_base = take(nblk * E * 4);
  L->counters = take((E + S + 2) * 4);   // per-group counters, the tile claim counter and
                                         // the exit ticket of a launch that zeroes them itself
  L->counters_s = take((S + 2) * 4);     // the same for a shared-experts-only launch, + its exit
                                         // ticket
  L->xperm = take(T * k * D * 2);
  L->act_r = take(T * k * F * 2);
  L->act_s = take(S * T * Fs * 2);
  L->y = take((T * k + S * T) * D * 4);
  L->touched = take(4);
  L->gmask = take(T <= kPermBlockTokens ? E * (kPermBlockTokens / 32) * 4 : 0);
  L->total = off;
  return true;
}

namespace {

// Expert weights of one call: bf16 matrices, or FP8 codes + exponents.
struct ExpertWeights {
  const uint16_t *W1 = nullptr, *W3 = nullptr, *W2 = nullptr, *Ws1 = nullptr, *Ws3 = nullptr,
                 *Ws2 = nullptr;
  bool fp8 = false;
  Fp8Weights f8{};
};

int check_bf16_weights(const void* W1, const void* W3, const void* W2, const void* Ws1,
                       const void* Ws3, const void* Ws2, const moe_dims_t* dims,
                       ExpertWeights* out) {
  MOE_CHECK_PTR(W1);
  MOE_CHECK_PTR(W3);
  MOE_CHECK_PTR(W2);
  if (dims->S > 0) {
    MOE_CHECK_PTR(Ws1);
    MOE_CHECK_PTR(Ws3);
    MOE_CHECK_PTR(Ws2);
  }
  out->W1 = static_cast<const uint16_t*>(W1);
  out->W3 = static_cast<const uint16_t*>(W3);
  out->W2 = static_cast<const uint16_t*>(W2);
  out->Ws1 = static_cast<const uint16_t*>(Ws1);
  out->Ws3 = static_cast<const uint16_t*>(Ws3);
  out->Ws2 = static_cast<const uint16_t*>(Ws2);
  out->fp8 = false;
  return MOE_OK;
}

// FP8 weight rows are D, F or Fs bytes long: TMA needs 16-byte row strides.
int check_fp8_dims(const moe_dims_t* d) {
  if (d->D % 16) return fail(MOE_ERR_INVALID_ARG, "FP8 weights: D = %d not a multiple of 16", d->D);
  if (d->F % 16) return fail(MOE_ERR_INVALID_ARG, "FP8 weights: F = %d not a multiple of 16", d->F);
  if (d->S > 0 && d->Fs % 16)
    return fail(MOE_ERR_INVALID_ARG, "FP8 weights: Fs = %d not a multiple of 16", d->Fs);
  return MOE_OK;
}

#define MOE_CHECK_EXP(p)                                                           \
  do {                                                                             \
    if (!(w8->p)) return fail(MOE_ERR_INVALID_ARG, "w8->%s is NULL", #p);          \
  } while (0)

int check_fp8_weights(const moe_fp8_weights_t* w8, const moe_dims_t* dims, ExpertWeights* out) {
  if (!w8) return fail(MOE_ERR_INVALID_ARG, "w8 is NULL");
  const void* W1 = w8->W1;
  const void* W3 = w8->W3;
  const void* W2 = w8->W2;
  MOE_CHECK_PTR(W1);
  MOE_CHECK_PTR(W3);
  MOE_CHECK_PTR(W2);
  MOE_CHECK_EXP(W1e);
  MOE_CHECK_EXP(W3e);
  MOE_CHECK_EXP(W2e);
  const int8_t *W1e = w8->W1e, *W3e = w8->W3e, *W2e = w8->W2e;
  const void *Ws1 = w8->Ws1, *Ws3 = w8->Ws3, *Ws2 = w8->Ws2;
  const int8_t *Ws1e = w8->Ws1e, *Ws3e = w8->Ws3e, *Ws2e = w8->Ws2e;
  if (dims->S > 0) {
    MOE_CHECK_PTR(Ws1);
    MOE_CHECK_PTR(Ws3);
    MOE_CHECK_PTR(Ws2);
    if (!Ws1e || !Ws3e || !Ws2e) return fail(MOE_ERR_INVALID_ARG, "w8->Ws*e is NULL with S > 0");
  }
  out->fp8 = true;
  out->f8.W1 = static_cast<const uint8_t*>(W1);
  out->f8.W3 = static_cast<const uint8_t*>(W3);
  out->f8.W2 = static_cast<const uint8_t*>(W2);
  out->f8.Ws1 = static_cast<const uint8_t*>(Ws1);
  out->f8.Ws3 = static_cast<const uint8_t*>(Ws3);
  out->f8.Ws2 = static_cast<const uint8_t*>(Ws2);
  out->f8.W1e = W1e; out->f8.W3e = W3e; out->f8.W2e = W2e;
  out->f8.Ws1e = Ws1e; out->f8.Ws3e = Ws3e; out->f8.Ws2e = Ws2e;
  return MOE_OK;
}

FfnArgs ffn_args(const uint16_t* h, const uint16_t* xperm, const int32_t* offsets,
                 const ExpertWeights& wt, const Ws& w, float* y, int32_t* counters,
                 const moe_dims_t* d) {
  FfnArgs a;
  a.xperm = xperm;
  a.h = h;
  a.offsets = offsets;
  a.W1 = wt.W1; a.W3 = wt.W3; a.W2 = wt.W2;
  a.Ws1 = wt.Ws1; a.Ws3 = wt.Ws3; a.Ws2 = wt.Ws2;
  a.act_r = w.at<uint16_t>(w.L.act_r);
  a.act_s = w.at<uint16_t>(w.L.act_s);
  a.y = y;
  a.status = w.status();
  a.counters = counters;
  a.T = d->T; a.D = d->D; a.E = d->E; a.F = d->F; a.k = d->k; a.S = d->S; a.Fs = d->Fs;
  return a;
}

cudaError_t launch_ffn(const FfnArgs& a, const ExpertWeights& wt, cudaStream_t st, int* n,
                       const char** why, void* const* marks) {
  return wt.fp8 ? launch_expert_ffn_fp8(a, wt.f8, st, n, why, marks)
                : launch_expert_ffn(a, st, n, why, marks);
}

int expert_ffn_impl(const void* h, const int32_t* perm, const int32_t* offsets,
                    const ExpertWeights& wt, const moe_dims_t* dims, float* y, void* ws,
                    size_t ws_bytes, moe_stream_t stream) {
  MOE_CHECK_PTR(h);
  MOE_CHECK_PTR(perm);
  MOE_CHECK_PTR(offsets);
  MOE_CHECK_PTR(y);
  Ws w;
  int rc;
  if ((rc = check_ws(dims, ws, ws_bytes, &w))) return rc;
  if ((rc = check_device())) return rc;
  const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int rows = dims->T * dims->k;
  const auto* hb = static_cast<const uint16_t*>(h);
  uint16_t* xperm = w.at<uint16_t>(w.L.xperm);
  int32_t* counters = w.at<int32_t>(w.L.counters);
  cudaError_t e = launch_gather_rows(hb, perm, rows, dims->D, dims->T, xperm, counters,
                                     dims->E + dims->S + 1, st);
  if (e != cudaSuccess) return cuda_fail(e, "gather launch");
  const FfnArgs a = ffn_args(hb, xperm, offsets, wt, w, y, counters, dims);
  int n = 1;
  const char* why = "launch failed";
  e = launch_ffn(a, wt, st, &n, &why, nullptr);
  if (e != cudaSuccess) return fail(MOE_ERR_CUDA, "expert ffn: %s (%s)", why, cudaGetErrorString(e));
  g_launches = n;
  return MOE_OK;
}

// An internal stream (per host thread and device) that runs the shared
// experts' FFN next to the routing, with the events that fork it from and join
// it to the caller's stream.  Created on first use, kept for the process.
struct SideStream {
  cudaStream_t s = nullptr;
  cudaEvent_t fork = nullptr, join = nullptr;
};

cudaError_t side_stream(SideStream** out) {
  thread_local SideStream per_dev[kMaxDev];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDev) return cudaErrorInvalidDevice;
  SideStream& r = per_dev[dev];
  if (!r.s) {
    // The highest priority: when the shared launch and the routing kernels
    // become ready together, the block scheduler places the shared CTAs
    // first, so the routed FFN launched behind them cannot take their SMs.
    int lo = 0, hi = 0;
    e = cudaDeviceGetStreamPriorityRange(&lo, &hi);
    if (e == cudaSuccess) e = cudaStreamCreateWithPriority(&r.s, cudaStreamNonBlocking, hi);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&r.fork, cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&r.join, cudaEventDisableTiming);
    if (e != cudaSuccess) {
      if (r.fork) cudaEventDestroy(r.fork);
      if (r.s) cudaStreamDestroy(r.s);
      r = SideStream{};
      return e;
    }
  }
  *out = &r;
  return cudaSuccess;
}

// Makes `st` wait for the side stream's join event when a forward returns
// early after forking, so that later work on `st` is ordered after the shared
// experts' kernels that read and write the workspace.
struct JoinGuard {
  cudaStream_t st = nullptr;
  cudaEvent_t join = nullptr;
  ~JoinGuard() {
    if (join) cudaStreamWaitEvent(st, join, 0);
  }
};

int forward_impl(const void* h, const float* Wr, const float* bias, const ExpertWeights& wt,
                 const moe_dims_t* dims, float* out, int32_t* idx_out, float* w_out, void* ws,
                 size_t ws_bytes, moe_stream_t stream) {
  MOE_CHECK_PTR(out);
  if (idx_out && !aligned16(idx_out)) return fail(MOE_ERR_INVALID_ARG, "idx_out is not 16-byte aligned");
  if (w_out && !aligned16(w_out)) return fail(MOE_ERR_INVALID_ARG, "w_out is not 16-byte aligned");
  Ws w;
  int rc;
  if ((rc = check_ws(dims, ws, ws_bytes, &w))) return rc;
  if ((rc = check_device())) return rc;
  const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int T = dims->T, D = dims->D, E = dims->E, k = dims->k;
  const auto* hb = static_cast<const uint16_t*>(h);
  int32_t* idx = idx_out ? idx_out : w.at<int32_t>(w.L.idx);
  float* rw = w_out ? w_out : w.at<float>(w.L.w);
  int32_t* counts = w.at<int32_t>(w.L.counts);
  int32_t* offsets = w.at<int32_t>(w.L.offsets);
  int32_t* perm = w.at<int32_t>(w.L.perm);
  int32_t* inv = w.at<int32_t>(w.L.inv);
  float* y = w.at<float>(w.L.y);
  int n = 0;

  const RouterSplit sp = router_split(T, D, E);
  float* partials = w.at<float>(w.L.partials);
  uint16_t* xperm = w.at<uint16_t>(w.L.xperm);
  int32_t* counters = w.at<int32_t>(w.L.counters);
  cudaError_t e = mark(0, st);
  if (e != cudaSuccess) return cuda_fail(e, "profile event");

  // Small batches: the shared experts need no routing, so their FFN runs on a
  // side stream on a few SMs while the routing kernels run here; the merge
  // waits for it.  Their weights then no longer lengthen the routed FFN.
  const bool overlap_shared = moe_forward_shared_overlap(dims, wt.fp8 ? 1 : 0) != 0;
  SideStream* side = nullptr;
  JoinGuard guard;
  if (overlap_shared) {
    e = side_stream(&side);
    if (e == cudaSuccess) e = cudaEventRecord(side->fork, st);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(side->s, side->fork, 0);
    // the shared launch's counters are zero: the workspace starts zeroed and
    // the launch's last CTA to finish zeroes them again
    int32_t* counters_s = w.at<int32_t>(w.L.counters_s);
    if (e != cudaSuccess) return cuda_fail(e, "shared-expert stream");
    FfnArgs as = ffn_args(hb, xperm, offsets, wt, w, y, counters, dims);
    as.part = kFfnShared;
    as.counters_s = counters_s;
    as.max_ctas = kSharedCtas;
    const char* swhy = "launch failed";
    e = launch_ffn(as, wt, side->s, &n, &swhy, nullptr);
    if (e != cudaSuccess)
      return fail(MOE_ERR_CUDA, "shared expert ffn: %s (%s)", swhy, cudaGetErrorString(e));
    e = cudaEventRecord(side->join, side->s);
    if (e != cudaSuccess) return cuda_fail(e, "shared-expert stream");
    guard.st = st;
    guard.join = side->join;
  }

  const char* rwhy = "router launch";
  if (e == cudaSuccess) e = launch_router(hb, Wr, *dims, sp, w, partials, st, &n, &rwhy);
  if (e == cudaSuccess) e = mark(1, st);
  if (e != cudaSuccess) return cuda_fail(e, rwhy);
  // Batches of at most 128 tokens with bf16 weights: the routed gate/up tiles
  // read the token matrix itself (one row tile holds the whole batch), so no
  // gathered copy is made.  No grouping pass runs either: the routing kernel
  // only sets each token's bit in the rows of its experts, and the FFN
  // derives the group offsets (and writes counts, offsets and inv) from
  // them; its last CTA zeroes its counters and the merge clears the bits.
  const bool dense = !wt.fp8 && T <= kDenseMaxT;
  uint32_t* gmask = w.at<uint32_t>(w.L.gmask);
  if (dense) {
    e = launch_route_bits(partials, sp.nsplit, bias, T, E, k, dims->scale, idx, rw, w.status(),
                          gmask, st);
    if (e == cudaSuccess) e = mark(2, st);
    if (e == cudaSuccess) e = mark(3, st);
    if (e != cudaSuccess) return cuda_fail(e, "route launch");
    n += 1;
  } else if (T <= kPermBlockTokens) {
    // small batches: the routing kernel's last block also groups the pairs
    const RouteGrouping grp{counts, offsets, perm, inv, w.at<int32_t>(w.L.touched),
                            w.at<int>(w.L.ticket), gmask};
    e = launch_route_and_group(partials, sp.nsplit, bias, T, E, k, dims->scale, idx, rw,
                               w.status(), grp, st);
    if (e == cudaSuccess) e = mark(2, st);
    if (e == cudaSuccess) e = mark(3, st);
    if (e != cudaSuccess) return cuda_fail(e, "route launch");
    n += 1;
  } else {
    e = launch_route(partials, sp.nsplit, bias, T, E, k, dims->scale, idx, rw, w.status(), st);
    if (e == cudaSuccess) e = mark(2, st);
    if (e != cudaSuccess) return cuda_fail(e, "route launch");
    n += 1;
    e = launch_permute(idx, T, E, k, counts, offsets, perm, inv, w.at<int32_t>(w.L.blk_base),
                       w.status(), w.at<int32_t>(w.L.touched), st, &n);
    if (e == cudaSuccess) e = mark(3, st);
    if (e != cudaSuccess) return cuda_fail(e, "permute launch");
  }
  if (!dense) {
    e = launch_gather_rows(hb, perm, T * k, D, T, xperm, counters, E + dims->S + 1, st);
    n += 1;
  }
  if (e == cudaSuccess) e = mark(4, st);
  if (e != cudaSuccess) return cuda_fail(e, "gather launch");
  FfnArgs a = ffn_args(hb, xperm, offsets, wt, w, y, counters, dims);
  if (overlap_shared) a.part = kFfnRouted;
  if (dense) {
    a.dense_a = 1;
    a.idx = idx;
    a.inv = inv;
    a.mask = gmask;
    a.mask_stride = kPermBlockTokens / 32;
    a.counts_out = counts;
    a.offsets_out = offsets;
    a.touched_out = w.at<int32_t>(w.L.touched);
    a.inv_out = inv;
    a.self_reset = 1;
  }
  const char* why = "launch failed";
  e = launch_ffn(a, wt, st, &n, &why, g_prof_events ? g_prof_events + 5 : nullptr);
  if (e != cudaSuccess) return fail(MOE_ERR_CUDA, "expert ffn: %s (%s)", why, cudaGetErrorString(e));
  // The merge reads the shared experts' rows: the streams are joined first.
  // (A device-side hand-off from the shared launch to the routed one would
  // let the merge launch behind the routed FFN, but a kernel that waits for
  // a kernel of another stream can wait for one that never becomes
  // resident.)
  if (overlap_shared) {
    guard.join = nullptr;
    e = cudaStreamWaitEvent(st, side->join, 0);
    if (e != cudaSuccess) return cuda_fail(e, "shared-expert stream");
  }
  e = launch_combine(y, rw, inv, T, D, k, dims->S, out, w.status(), dense ? idx : nullptr,
                     dense ? gmask : nullptr, kPermBlockTokens / 32, st);
  if (e == cudaSuccess) e = mark(6, st);
  if (e != cudaSuccess) return cuda_fail(e, "combine launch");
  n += 1;
  g_launches = n;
  return MOE_OK;
}

// Device memory of a host-buffer pipeline: two input slots, two output slots
// and the layer's workspace, each 256-byte aligned.
struct PipeLayout {
  size_t h[2], out[2], ws, ws_bytes, total;
};

bool pipe_layout(const moe_dims_t& d, PipeLayout* L) {
  WsLayout W;
  if (!ws_layout(d, &W)) return false;
  const size_t hb = align256((size_t)d.T * d.D * 2), ob = align256((size_t)d.T * d.D * 4);
  size_t off = 0;
  for (int s = 0; s < 2; ++s) { L->h[s] = off; off += hb; }
  for (int s = 0; s < 2; ++s) { L->out[s] = off; off += ob; }
  L->ws = off;
  L->ws_bytes = W.total;
  L->total = off + align256(W.total);
  return true;
}

// Host pointers the pipeline copies from or to must be page-locked: a copy
// from pageable memory is staged by the driver and cannot overlap the layer.
int check_pinned(const void* p, const char* name) {
  if (!p) return fail(MOE_ERR_INVALID_ARG, "%s is NULL", name);
  cudaPointerAttributes a;
  cudaError_t e = cudaPointerGetAttributes(&a, p);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(MOE_ERR_INVALID_ARG, "%s: %s", name, cudaGetErrorString(e));
  }
  if (a.type != cudaMemoryTypeHost)
    return fail(MOE_ERR_INVALID_ARG, "%s is not page-locked host memory", name);
  return MOE_OK;
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" {

size_t moe_workspace_size(const moe_dims_t* dims) {
  if (check_dims(dims) != MOE_OK) return 0;
  WsLayout L;
  ws_layout(*dims, &L);
  return L.total;
}

const char* moe_last_error(void) { return g_err.c_str(); }

int moe_last_launch_count(void) { return g_launches; }

int moe_forward_shared_overlap(const moe_dims_t* dims, int fp8_weights) {
  if (check_dims(dims) != MOE_OK || fp8_weights) return 0;
  const double shared_bytes = 3.0 * dims->S * (double)dims->Fs * dims->D * 2;
  return dims->S > 0 && dims->T > 0 && dims->T <= kOverlapSharedMaxT &&
                 shared_bytes >= kOverlapSharedMinBytes
             ? 1
             : 0;
}

int moe_set_profile_events(void* const* events, int n) {
  g_err.clear();
  if (n == 0) {
    g_prof_events = nullptr;
    return MOE_OK;
  }
  if (n != MOE_PROFILE_EVENTS || !events)
    return fail(MOE_ERR_INVALID_ARG, "profile events: need %d event handles", MOE_PROFILE_EVENTS);
  for (int i = 0; i < n; ++i)
    if (!events[i]) return fail(MOE_ERR_INVALID_ARG, "profile event %d is NULL", i);
  g_prof_events = events;
  return MOE_OK;
}

int moe_router_logits(const void* h, const float* Wr, const moe_dims_t* dims, float* logits,
                      void* ws, size_t ws_bytes, moe_stream_t stream) {
  int rc = begin(dims);
  if (rc) return rc;
  if (dims->T == 0) return MOE_OK;
  MOE_CHECK_PTR(h);
  MOE_CHECK_PTR(Wr);
  MOE_CHECK_PTR(logits);
  const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const RouterSplit sp = router_split(dims->T, dims->D, dims->E);
  Ws w{};
  if ((sp.nsplit > 1 || sp.tensor) && (rc = check_ws(dims, ws, ws_bytes, &w))) return rc;
  if ((rc = check_device())) return rc;
  float* dst = sp.nsplit == 1 ? logits : w.at<float>(w.L.partials);
  int n = 0;
  const char* why = "router launch";
  cudaError_t e = launch_router(static_cast<const uint16_t*>(h), Wr, *dims, sp, w, dst, st, &n, &why);
  if (e != cudaSuccess) return cuda_fail(e, why);
  if (sp.nsplit > 1) {
    e = launch_reduce_partials(dst, sp.nsplit, (size_t)dims->T * dims->E, logits, st);
    if (e != cudaSuccess) return cuda_fail(e, "router reduce launch");
    n += 1;
  }
  g_launches = n;
  return MOE_OK;
}

int moe_route(const float* logits, const float* bias, const moe_dims_t* dims, int32_t* idx,
              float* w, void* ws, moe_stream_t stream) {
  int rc = begin(dims);
  if (rc) return rc;
  if (dims->T == 0) return MOE_OK;
  MOE_CHECK_PTR(logits);
  MOE_CHECK_PTR(bias);
  MOE_CHECK_PTR(idx);
  MOE_CHECK_PTR(w);
  if (ws && (reinterpret_cast<uintptr_t>(ws) & 255u))
    return fail(MOE_ERR_WORKSPACE, "workspace is not 256-byte aligned");
  WsLayout L;
  ws_layout(*dims, &L);
  int* status = ws ? reinterpret_cast<int*>(static_cast<uint8_t*>(ws) + L.status) : nullptr;
  if ((rc = check_device())) return rc;
  cudaError_t e = launch_route(logits, 1, bias, dims->T, dims->E, dims->k, dims->scale, idx, w,
                               status, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "route launch");
  g_launches = 1;
  return MOE_OK;
}

int moe_route_grouped(const float* logits, const float* bias, const moe_dims_t* dims, int n_group,
                      int topk_group, int32_t* idx, float* w, void* ws, moe_stream_t stream) {
  int rc = begin(dims);
  if (rc) return rc;
  if (n_group < 1 || n_group > 32 || dims->E % n_group)
    return fail(MOE_ERR_INVALID_ARG, "n_group = %d must divide E = %d and be in [1, 32]", n_group,
                dims->E);
  if (topk_group < 1 || topk_group > n_group)
    return fail(MOE_ERR_INVALID_ARG, "topk_group = %d outside [1, n_group]", topk_group);
  if ((long long)dims->k > (long long)topk_group * (dims->E / n_group))
    return fail(MOE_ERR_INVALID_ARG, "k = %d exceeds the %d experts of the kept groups", dims->k,
                topk_group * (dims->E / n_group));
  if (dims->T == 0) return MOE_OK;
  MOE_CHECK_PTR(logits);
  MOE_CHECK_PTR(bias);
  MOE_CHECK_PTR(idx);
  MOE_CHECK_PTR(w);
  if (ws && (reinterpret_cast<uintptr_t>(ws) & 255u))
    return fail(MOE_ERR_WORKSPACE, "workspace is not 256-byte aligned");
  WsLayout L;
  ws_layout(*dims, &L);
  int* status = ws ? reinterpret_cast<int*>(static_cast<uint8_t*>(ws) + L.status) : nullptr;
  if ((rc = check_device())) return rc;
  cudaError_t e = launch_route_grouped(logits, bias, dims->T, dims->E, dims->k, dims->scale, n_group,
                                       topk_group, idx, w, status,
                                       reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "grouped route launch");
  g_launches = 1;
  return MOE_OK;
}

int moe_permute(const int32_t* idx, const moe_dims_t* dims, int32_t* counts, int32_t* offsets,
                int32_t* perm, int32_t* inv, void* ws, size_t ws_bytes, moe_stream_t stream) {
  int rc = begin(dims);
  if (rc) return rc;
  MOE_CHECK_PTR(counts);
  MOE_CHECK_PTR(offsets);
  const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (dims->T == 0) {
    if ((rc = check_device())) return rc;
    // no pairs: every count and offset is zero
    cudaError_t e = cudaMemsetAsync(counts, 0, (size_t)dims->E * 4, st);
    if (e == cudaSuccess) e = cudaMemsetAsync(offsets, 0, (size_t)(dims->E + 1) * 4, st);
    if (e != cudaSuccess) return cuda_fail(e, "memset");
    return MOE_OK;
  }
  MOE_CHECK_PTR(idx);
  MOE_CHECK_PTR(perm);
  MOE_CHECK_PTR(inv);
  Ws w;
  if ((rc = check_ws(dims, ws, ws_bytes, &w))) return rc;
  if ((rc = check_device())) return rc;
  int n = 0;
  cudaError_t e = launch_permute(idx, dims->T, dims->E, dims->k, counts, offsets, perm, inv,
                                 w.at<int32_t>(w.L.blk_base), w.status(),
                                 w.at<int32_t>(w.L.touched), st, &n);
  if (e != cudaSuccess) return cuda_fail(e, "permute launch");
  g_launches = n;
  return MOE_OK;
}

int moe_permute_noalloc(const int32_t* idx, const moe_dims_t* dims, int32_t* counts,
                        int32_t* offsets, int32_t* perm, int32_t* inv, moe_stream_t stream) {
  int rc = begin(dims);
  if (rc) return rc;
  MOE_CHECK_PTR(counts);
  MOE_CHECK_PTR(offsets);
  const int nblk = (dims->T + kPermBlockTokens - 1) / kPermBlockTokens;
  if (nblk > kNoAllocMaxBlocks || dims->E > kNoAllocMaxExperts)
    return fail(MOE_ERR_UNSUPPORTED,
                "moe_permute_noalloc: T = %d, E = %d exceeds the static scratch (T <= %d, E <= %d)",
                dims->T, dims->E, kNoAllocMaxBlocks * kPermBlockTokens, kNoAllocMaxExperts);
  const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (dims->T == 0) {
    if ((rc = check_device())) return rc;
    cudaError_t e = cudaMemsetAsync(counts, 0, (size_t)dims->E * 4, st);
    if (e == cudaSuccess) e = cudaMemsetAsync(offsets, 0, (size_t)(dims->E + 1) * 4, st);
    if (e != cudaSuccess) return cuda_fail(e, "memset");
    return MOE_OK;
  }
  MOE_CHECK_PTR(idx);
  MOE_CHECK_PTR(perm);
  MOE_CHECK_PTR(inv);
  if ((rc = check_device())) return rc;
  int32_t* scratch = nullptr;
  cudaError_t e = noalloc_scratch(&scratch);
  if (e != cudaSuccess) return cuda_fail(e, "moe_permute_noalloc: scratch address lookup");
  int n = 0;
  e = launch_permute(idx, dims->T, dims->E, dims->k, counts, offsets, perm, inv, scratch,
                     nullptr, nullptr, st, &n);
  if (e != cudaSuccess) return cuda_fail(e, "permute launch");
  g_launches = n;
  return MOE_OK;
}

int moe_expert_ffn(const void* h, const int32_t* perm, const int32_t* offsets, const void* W1,
                   const void* W3, const void* W2, const void* Ws1, const void* Ws3,
                   const void* Ws2, const moe_dims_t* dims, float* y, void* ws, size_t ws_bytes,
                   moe_stream_t stream) {
  int rc = begin(dims);
  if (rc) return rc;
  if (dims->T == 0) return MOE_OK;
  ExpertWeights wt;
  if ((rc = check_bf16_weights(W1, W3, W2, Ws1, Ws3, Ws2, dims, &wt))) return rc;
  return expert_ffn_impl(h, perm, offsets, wt, dims, y, ws, ws_bytes, stream);
}

int moe_expert_ffn_fp8(const void* h, const int32_t* perm, const int32_t* offsets,
                       const moe_fp8_weights_t* w8, const moe_dims_t* dims, float* y, void* ws,
                       size_t ws_bytes, moe_stream_t stream) {
  int rc = begin(dims);
  if (rc) return rc;
  if ((rc = check_fp8_dims(dims))) return rc;
  if (dims->T == 0) return MOE_OK;
  ExpertWeights wt;
  if ((rc = check_fp8_weights(w8, dims, &wt))) return rc;
  return expert_ffn_impl(h, perm, offsets, wt, dims, y, ws, ws_bytes, stream);
}

int moe_combine(const float* y, const float* w, const int32_t* inv, const moe_dims_t* dims,
                float* out, void* ws, moe_stream_t stream) {
  int rc = begin(dims);
  if (rc) return rc;
  if (dims->T == 0) return MOE_OK;
  MOE_CHECK_PTR(y);
  MOE_CHECK_PTR(w);
  MOE_CHECK_PTR(inv);
  MOE_CHECK_PTR(out);
  if (ws && (reinterpret_cast<uintptr_t>(ws) & 255u))
    return fail(MOE_ERR_WORKSPACE, "workspace is not 256-byte aligned");
  WsLayout L;
  ws_layout(*dims, &L);
  int* status = ws ? reinterpret_cast<int*>(static_cast<uint8_t*>(ws) + L.status) : nullptr;
  if ((rc = check_device())) return rc;
  cudaError_t e = launch_combine(y, w, inv, dims->T, dims->D, dims->k, dims->S,
                                 out, status, nullptr, nullptr, 0,
                                 reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "combine launch");
  g_launches = 1;
  return MOE_OK;
}

int moe_forward(const void* h, const float* Wr, const float* bias, const void* W1,
                const void* W3, const void* W2, const void* Ws1, const void* Ws3,
                const void* Ws2, const moe_dims_t* dims, float* out, int32_t* idx_out,
                float* w_out, void* ws, size_t ws_bytes, moe_stream_t stream) {
  int rc = begin(dims);
  if (rc) return rc;
  if (dims->T == 0) return MOE_OK;
  MOE_CHECK_PTR(h);
  MOE_CHECK_PTR(Wr);
  MOE_CHECK_PTR(bias);
  ExpertWeights wt;
  if ((rc = check_bf16_weights(W1, W3, W2, Ws1, Ws3, Ws2, dims, &wt))) return rc;
  return forward_impl(h, Wr, bias, wt, dims, out, idx_out, w_out, ws, ws_bytes, stream);
}

int moe_forward_fp8(const void* h, const float* Wr, const float* bias, const moe_fp8_weights_t* w8,
                    const moe_dims_t* dims, float* out, int32_t* idx_out, float* w_out, void* ws,
                    size_t ws_bytes, moe_stream_t stream) {
  int rc = begin(dims);
  if (rc) return rc;
  if ((rc = check_fp8_dims(dims))) return rc;
  if (dims->T == 0) return MOE_OK;
  MOE_CHECK_PTR(h);
  MOE_CHECK_PTR(Wr);
  MOE_CHECK_PTR(bias);
  ExpertWeights wt;
  if ((rc = check_fp8_weights(w8, dims, &wt))) return rc;
  return forward_impl(h, Wr, bias, wt, dims, out, idx_out, w_out, ws, ws_bytes, stream);
}

int moe_fp8_dequantize(const void* codes, const int8_t* exps, int G, int R, int K, void* out,
                       void* ws, moe_stream_t stream) {
  g_err.clear();
  g_launches = 0;
  if (G < 0 || R < 0 || K < 0) return fail(MOE_ERR_INVALID_ARG, "G, R, K must be >= 0");
  if (K % 16) return fail(MOE_ERR_INVALID_ARG, "K = %d is not a multiple of 16", K);
  if ((long long)G * R * K >= (1ll << 40)) return fail(MOE_ERR_UNSUPPORTED, "G*R*K >= 2^40");
  if ((long long)G * R * K == 0) return MOE_OK;
  MOE_CHECK_PTR(codes);
  MOE_CHECK_PTR(out);
  if (!exps) return fail(MOE_ERR_INVALID_ARG, "exps is NULL");
  if (ws && (reinterpret_cast<uintptr_t>(ws) & 255u))
    return fail(MOE_ERR_WORKSPACE, "workspace is not 256-byte aligned");
  int rc = check_device();
  if (rc) return rc;
  cudaError_t e = launch_fp8_dequantize(static_cast<const uint8_t*>(codes), exps, G, R, K,
                                        static_cast<uint16_t*>(out), static_cast<int*>(ws),
                                        reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "dequantize launch");
  g_launches = 1;
  return MOE_OK;
}

int moe_gather_rows(const void* src, int src_rows, const int32_t* idx, int n, int row_bytes,
                    void* dst, void* ws, moe_stream_t stream) {
  g_err.clear();
  g_launches = 0;
  if (src_rows < 0 || n < 0) return fail(MOE_ERR_INVALID_ARG, "src_rows and n must be >= 0");
  if (row_bytes <= 0 || row_bytes % 16)
    return fail(MOE_ERR_INVALID_ARG, "row_bytes = %d is not a positive multiple of 16", row_bytes);
  if (n == 0) return MOE_OK;
  MOE_CHECK_PTR(src);
  MOE_CHECK_PTR(idx);
  MOE_CHECK_PTR(dst);
  if (ws && (reinterpret_cast<uintptr_t>(ws) & 255u))
    return fail(MOE_ERR_WORKSPACE, "workspace is not 256-byte aligned");
  int rc = check_device();
  if (rc) return rc;
  cudaError_t e = launch_gather_bytes(src, src_rows, idx, n, row_bytes, dst, static_cast<int*>(ws),
                                      reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "gather launch");
  g_launches = 1;
  return MOE_OK;
}

const int32_t* moe_ws_expert_counts(const void* ws, const moe_dims_t* dims) {
  if (!ws || check_dims(dims) != MOE_OK) return nullptr;
  WsLayout L;
  ws_layout(*dims, &L);
  return reinterpret_cast<const int32_t*>(static_cast<const uint8_t*>(ws) + L.counts);
}

const int32_t* moe_ws_touched_experts(const void* ws, const moe_dims_t* dims) {
  if (!ws || check_dims(dims) != MOE_OK) return nullptr;
  WsLayout L;
  ws_layout(*dims, &L);
  return reinterpret_cast<const int32_t*>(static_cast<const uint8_t*>(ws) + L.touched);
}

int moe_selftest_bounded_wait(void* ws, moe_stream_t stream) {
  g_err.clear();
  g_launches = 0;
  if (!ws) return fail(MOE_ERR_INVALID_ARG, "workspace is NULL");
  if (reinterpret_cast<uintptr_t>(ws) & 255u)
    return fail(MOE_ERR_WORKSPACE, "workspace is not 256-byte aligned");
  int rc = check_device();
  if (rc) return rc;
  cudaError_t e = launch_bounded_wait_selftest(static_cast<int*>(ws),
                                               reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "self-test launch");
  g_launches = 1;
  return MOE_OK;
}

int moe_selftest_occupy(int nctas, long long cycles, moe_stream_t stream) {
  g_err.clear();
  g_launches = 0;
  int rc = check_device();
  if (rc) return rc;
  if (nctas < 1 || nctas > num_sms())
    return fail(MOE_ERR_INVALID_ARG, "nctas = %d outside [1, %d]", nctas, num_sms());
  if (cycles < 0 || cycles > kOccupyMaxCycles)
    return fail(MOE_ERR_INVALID_ARG, "cycles = %lld outside [0, %lld]", cycles, kOccupyMaxCycles);
  cudaError_t e = launch_occupy_selftest(nctas, cycles, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "occupy self-test launch");
  g_launches = 1;
  return MOE_OK;
}

int moe_get_device_status(void* ws, moe_stream_t stream) {
  g_err.clear();
  if (!ws) return fail(MOE_ERR_INVALID_ARG, "workspace is NULL");
  const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  int word = 0;
  cudaError_t e = cudaMemcpyAsync(&word, ws, sizeof(int), cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e == cudaSuccess) e = cudaMemsetAsync(ws, 0, sizeof(int), st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(e, "reading the device status word");
  if (word & kStNonFinite) return fail(MOE_ERR_NONFINITE, "device: non-finite router logit or key");
  if (word & kStBounds)
    return fail(MOE_ERR_BOUNDS, "device: expert index, group offset or row index out of range");
  if (word & kStTimeout) return fail(MOE_ERR_TIMEOUT, "device: a bounded wait gave up");
  return MOE_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Host-buffer pipeline
// ---------------------------------------------------------------------------
// Step n uses slot n % 2.  Before its input copy overwrites input slot s, the
// copy stream waits for step n-2's layer (which read that slot); before its
// layer overwrites output slot s, the compute stream waits for step n-2's
// output copy.  Events never recorded count as complete, so the first two
// steps wait on nothing.
struct moe_pipeline {
  moe_dims_t dims{};
  moe::ExpertWeights wt{};
  const float* Wr = nullptr;
  const float* bias = nullptr;
  void* h_dev[2] = {nullptr, nullptr};
  float* out_dev[2] = {nullptr, nullptr};
  void* ws = nullptr;
  size_t ws_bytes = 0;
  cudaStream_t compute = nullptr, copy_in = nullptr, copy_out = nullptr;
  cudaEvent_t in_done[2] = {nullptr, nullptr};
  cudaEvent_t layer_done[2] = {nullptr, nullptr};
  cudaEvent_t out_done[2] = {nullptr, nullptr};
  long long steps = 0;
  int device = 0;
};

namespace {

// Waits for the pipeline's outstanding work and frees its streams and
// events; returns the first CUDA error met.
cudaError_t pipeline_release(moe_pipeline* p) {
  cudaError_t first = cudaSuccess;
  auto keep = [&first](cudaError_t e) {
    if (first == cudaSuccess && e != cudaSuccess) first = e;
  };
  if (p->copy_in) keep(cudaStreamSynchronize(p->copy_in));
  for (int s = 0; s < 2; ++s)
    if (p->layer_done[s]) keep(cudaEventSynchronize(p->layer_done[s]));
  if (p->copy_out) keep(cudaStreamSynchronize(p->copy_out));
  for (int s = 0; s < 2; ++s) {
    if (p->in_done[s]) keep(cudaEventDestroy(p->in_done[s]));
    if (p->layer_done[s]) keep(cudaEventDestroy(p->layer_done[s]));
    if (p->out_done[s]) keep(cudaEventDestroy(p->out_done[s]));
  }
  if (p->copy_in) keep(cudaStreamDestroy(p->copy_in));
  if (p->copy_out) keep(cudaStreamDestroy(p->copy_out));
  delete p;
  return first;
}

}  // namespace

extern "C" {

size_t moe_pipeline_device_bytes(const moe_dims_t* dims) {
  if (check_dims(dims) != MOE_OK) return 0;
  PipeLayout L;
  if (!pipe_layout(*dims, &L)) return 0;
  return L.total;
}

int moe_pipeline_create(const moe_dims_t* dims, const float* Wr, const float* bias,
                        const void* W1, const void* W3, const void* W2, const void* Ws1,
                        const void* Ws3, const void* Ws2, const moe_fp8_weights_t* w8,
                        void* dev, size_t dev_bytes, moe_stream_t stream, moe_pipeline_t** out) {
  if (out) *out = nullptr;
  int rc = begin(dims);
  if (rc) return rc;
  if (!out) return fail(MOE_ERR_INVALID_ARG, "out is NULL");
  MOE_CHECK_PTR(Wr);
  MOE_CHECK_PTR(bias);
  ExpertWeights wt;
  if (w8) {
    if ((rc = check_fp8_dims(dims))) return rc;
    if ((rc = check_fp8_weights(w8, dims, &wt))) return rc;
  } else if ((rc = check_bf16_weights(W1, W3, W2, Ws1, Ws3, Ws2, dims, &wt))) {
    return rc;
  }
  PipeLayout L;
  if (!pipe_layout(*dims, &L)) return fail(MOE_ERR_INVALID_ARG, "pipeline layout overflow");
  if (!dev) return fail(MOE_ERR_WORKSPACE, "dev is NULL");
  if (reinterpret_cast<uintptr_t>(dev) & 255u)
    return fail(MOE_ERR_WORKSPACE, "dev is not 256-byte aligned");
  if (dev_bytes < L.total)
    return fail(MOE_ERR_WORKSPACE, "dev has %zu bytes, needs %zu", dev_bytes, L.total);
  if ((rc = check_device())) return rc;

  moe_pipeline* p = new (std::nothrow) moe_pipeline();
  if (!p) return fail(MOE_ERR_UNSUPPORTED, "out of host memory");
  p->dims = *dims;
  p->wt = wt;
  p->Wr = Wr;
  p->bias = bias;
  uint8_t* base = static_cast<uint8_t*>(dev);
  for (int s = 0; s < 2; ++s) {
    p->h_dev[s] = base + L.h[s];
    p->out_dev[s] = reinterpret_cast<float*>(base + L.out[s]);
  }
  p->ws = base + L.ws;
  p->ws_bytes = L.ws_bytes;
  p->compute = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = cudaGetDevice(&p->device);
  if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&p->copy_in, cudaStreamNonBlocking);
  if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&p->copy_out, cudaStreamNonBlocking);
  for (int s = 0; s < 2 && e == cudaSuccess; ++s) {
    e = cudaEventCreateWithFlags(&p->in_done[s], cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&p->layer_done[s], cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&p->out_done[s], cudaEventDisableTiming);
  }
  // the workspace starts zeroed (status word and counters)
  if (e == cudaSuccess) e = cudaMemsetAsync(p->ws, 0, p->ws_bytes, p->compute);
  if (e != cudaSuccess) {
    pipeline_release(p);
    return cuda_fail(e, "pipeline create");
  }
  *out = p;
  return MOE_OK;
}

int moe_pipeline_submit(moe_pipeline_t* p, const void* h_host, float* out_host) {
  g_err.clear();
  g_launches = 0;
  if (!p) return fail(MOE_ERR_INVALID_ARG, "pipeline is NULL");
  if (p->dims.T == 0) return MOE_OK;  // nothing to copy or compute
  int rc;
  if ((rc = check_pinned(h_host, "h_host"))) return rc;
  if ((rc = check_pinned(out_host, "out_host"))) return rc;
  int cur = 0;
  cudaError_t e = cudaGetDevice(&cur);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (cur != p->device)
    return fail(MOE_ERR_INVALID_ARG, "current device %d is not the pipeline's device %d", cur,
                p->device);
  const int s = static_cast<int>(p->steps & 1);
  const size_t hb = (size_t)p->dims.T * p->dims.D * 2, ob = (size_t)p->dims.T * p->dims.D * 4;
  e = cudaStreamWaitEvent(p->copy_in, p->layer_done[s], 0);
  if (e == cudaSuccess)
    e = cudaMemcpyAsync(p->h_dev[s], h_host, hb, cudaMemcpyHostToDevice, p->copy_in);
  if (e == cudaSuccess) e = cudaEventRecord(p->in_done[s], p->copy_in);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(p->compute, p->in_done[s], 0);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(p->compute, p->out_done[s], 0);
  if (e != cudaSuccess) return cuda_fail(e, "pipeline input copy");
  rc = forward_impl(p->h_dev[s], p->Wr, p->bias, p->wt, &p->dims, p->out_dev[s], nullptr, nullptr,
                    p->ws, p->ws_bytes, reinterpret_cast<moe_stream_t>(p->compute));
  if (rc) return rc;
  const int n = g_launches;
  e = cudaEventRecord(p->layer_done[s], p->compute);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(p->copy_out, p->layer_done[s], 0);
  if (e == cudaSuccess)
    e = cudaMemcpyAsync(out_host, p->out_dev[s], ob, cudaMemcpyDeviceToHost, p->copy_out);
  if (e == cudaSuccess) e = cudaEventRecord(p->out_done[s], p->copy_out);
  if (e != cudaSuccess) return cuda_fail(e, "pipeline output copy");
  ++p->steps;
  g_launches = n;
  return MOE_OK;
}

int moe_pipeline_wait(moe_pipeline_t* p) {
  g_err.clear();
  if (!p) return fail(MOE_ERR_INVALID_ARG, "pipeline is NULL");
  cudaError_t e = cudaStreamSynchronize(p->copy_in);
  for (int s = 0; s < 2 && e == cudaSuccess; ++s) e = cudaEventSynchronize(p->layer_done[s]);
  if (e == cudaSuccess) e = cudaStreamSynchronize(p->copy_out);
  if (e != cudaSuccess) return cuda_fail(e, "pipeline wait");
  return moe_get_device_status(p->ws, reinterpret_cast<moe_stream_t>(p->compute));
}

int moe_pipeline_destroy(moe_pipeline_t* p) {
  g_err.clear();
  if (!p) return MOE_OK;
  const cudaError_t e = pipeline_release(p);
  return e == cudaSuccess ? MOE_OK : cuda_fail(e, "pipeline destroy");
}

}  // extern "C"
