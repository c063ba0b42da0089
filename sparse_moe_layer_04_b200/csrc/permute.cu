// Grouping of (token, slot) pairs by expert: a counting sort over blocks of
// tokens.  The pages name the expert kernels "grouped" ("GLM-5.2", PocketLLM,
// Implemented execution path); the grouping itself is the plain counting sort
// that makes each expert's rows contiguous.
//
//   count   : per block of 256 tokens, per-expert counts (shared atomics)
//   scan    : per-expert running sums over blocks, then an exclusive scan over
//             experts -> counts, offsets and each block's base row per expert
//   scatter : a per-block bitmask of the tokens that chose each expert gives
//             every pair its rank among the block's tokens for that expert
//             (tokens pick distinct experts, so one bit per token suffices):
//             row = base[block][e] + rank.  Rows within an expert therefore
//             follow increasing token order, i.e. (token, slot) order.
// Batches of at most 256 tokens (one counting block) run all three phases in
// one launch.  All integer work: exact and deterministic.
#include <atomic>

#include "moe_internal.cuh"
#include "permute_block.cuh"
#include "sm100_ptx.cuh"

namespace moe {

constexpr int kWordsPerBlock = kPermWords;

__global__ void __launch_bounds__(kPermBlockTokens) permute_count_kernel(
    const int32_t* __restrict__ idx, int T, int E, int k, int32_t* __restrict__ blk_counts,
    int* __restrict__ status) {
  ptx::pdl_launch_dependents();
  ptx::pdl_wait();
  extern __shared__ int cnt[];
  for (int e = threadIdx.x; e < E; e += blockDim.x) cnt[e] = 0;
  __syncthreads();
  const int t = blockIdx.x * kPermBlockTokens + threadIdx.x;
  bool bad = false;
  if (t < T) {
    for (int j = 0; j < k; ++j) {
      const int e = idx[(size_t)t * k + j];
      if (e < 0 || e >= E) {
        bad = true;
        continue;
      }
      atomicAdd(&cnt[e], 1);
    }
  }
  if (bad && status) atomicOr(status, kStBounds);
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x)
    blk_counts[(size_t)blockIdx.x * E + e] = cnt[e];
}

// One block of 1024 threads: thread e owns expert e (E <= 1024).
__global__ void __launch_bounds__(1024) permute_scan_kernel(int32_t* __restrict__ blk_base,
                                                            int nblk, int E,
                                                            int32_t* __restrict__ counts,
                                                            int32_t* __restrict__ offsets,
                                                            int32_t* __restrict__ touched) {
  ptx::pdl_launch_dependents();
  ptx::pdl_wait();
  __shared__ int warp_sums[32];
  const int e = threadIdx.x;
  int total = 0;
  if (e < E) {
    for (int b = 0; b < nblk; ++b) {
      const int c = blk_base[(size_t)b * E + e];
      blk_base[(size_t)b * E + e] = total;  // exclusive within the expert
      total += c;
    }
    counts[e] = total;
  }
  // exclusive scan of `total` over e
  const int lane = e & 31, wid = e >> 5;
  int incl = total;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += v;
  }
  if (lane == 31) warp_sums[wid] = incl;
  __syncthreads();
  if (wid == 0) {
    int v = warp_sums[lane];
    int s = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int u = __shfl_up_sync(0xffffffffu, s, off);
      if (lane >= off) s += u;
    }
    warp_sums[lane] = s - v;  // exclusive over warps
  }
  __syncthreads();
  const int excl = incl - total + warp_sums[wid];
  if (e < E) {
    offsets[e] = excl;
    if (e == E - 1) offsets[E] = excl + total;
    for (int b = 0; b < nblk; ++b) blk_base[(size_t)b * E + e] += excl;
  }
  const int nz = __syncthreads_count(e < E && total > 0);
  if (touched && e == 0) *touched = nz;
}

__global__ void __launch_bounds__(kPermBlockTokens) permute_scatter_kernel(
    const int32_t* __restrict__ idx, int T, int E, int k, const int32_t* __restrict__ blk_base,
    int32_t* __restrict__ perm, int32_t* __restrict__ inv, int* __restrict__ status) {
  ptx::pdl_launch_dependents();
  ptx::pdl_wait();
  extern __shared__ unsigned mask[];  // [E][kWordsPerBlock]
  for (int i = threadIdx.x; i < E * kWordsPerBlock; i += blockDim.x) mask[i] = 0u;
  __syncthreads();
  const int tl = threadIdx.x;
  const int t = blockIdx.x * kPermBlockTokens + tl;
  const int word = tl >> 5;
  const unsigned bit = 1u << (tl & 31);
  bool bad = false;
  if (t < T) {
    for (int j = 0; j < k; ++j) {
      const int e = idx[(size_t)t * k + j];
      if (e < 0 || e >= E) {
        bad = true;
        continue;
      }
      const unsigned old = atomicOr(&mask[e * kWordsPerBlock + word], bit);
      if (old & bit) bad = true;  // the same expert twice in one token
    }
  }
  __syncthreads();
  if (t < T && !bad) {
    for (int j = 0; j < k; ++j) {
      const int e = idx[(size_t)t * k + j];
      const unsigned* m = mask + e * kWordsPerBlock;
      int rank = __popc(m[word] & (bit - 1u));
      for (int q = 0; q < word; ++q) rank += __popc(m[q]);
      const int row = blk_base[(size_t)blockIdx.x * E + e] + rank;
      perm[row] = t;
      inv[(size_t)t * k + j] = row;
    }
  }
  if (bad && status) atomicOr(status, kStBounds);
}

// All three phases for T <= 256 in one block of 256 threads.
__global__ void __launch_bounds__(kPermBlockTokens) permute_single_block_kernel(
    const int32_t* __restrict__ idx, int T, int E, int k, int32_t* __restrict__ counts,
    int32_t* __restrict__ offsets, int32_t* __restrict__ perm, int32_t* __restrict__ inv,
    int* __restrict__ status, int32_t* __restrict__ touched) {
  ptx::pdl_launch_dependents();
  ptx::pdl_wait();
  extern __shared__ int sm[];
  permute_block(idx, T, E, k, counts, offsets, perm, inv, status, touched, sm);
}

// ---------------------------------------------------------------------------
// Scratch for the allocation-free variant of the grouping.  It lives in the
// library's own device memory, so callers that cannot allocate device memory
// still get the multi-block path.  Every GPU that loads the library holds it
// until the process exits.
// ---------------------------------------------------------------------------
static __device__ __align__(256) int32_t g_perm_scratch[kNoAllocMaxBlocks * kNoAllocMaxExperts];

// Device address of the scratch array on the current device.  Host code only
// sees a stand-in symbol for a __device__ array, so the address is looked up
// with cudaGetSymbolAddress, once per device, with that device current.  The
// cache is one atomic pointer per device: host threads whose first calls race
// may each look the address up, and they store the same value.
cudaError_t noalloc_scratch(int32_t** out) {
  constexpr int kMaxDevices = 64;
  static std::atomic<int32_t*> addr[kMaxDevices];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  int32_t* a = addr[dev].load(std::memory_order_acquire);
  if (!a) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_perm_scratch);
    if (e != cudaSuccess) return e;
    a = static_cast<int32_t*>(p);
    addr[dev].store(a, std::memory_order_release);
  }
  *out = a;
  return cudaSuccess;
}

cudaError_t launch_permute(const int32_t* idx, int T, int E, int k, int32_t* counts,
                           int32_t* offsets, int32_t* perm, int32_t* inv, int32_t* blk_base,
                           int* status, int32_t* touched, cudaStream_t st, int* nlaunch) {
  const int nblk = (T + kPermBlockTokens - 1) / kPermBlockTokens;
  if (nblk == 1) {
    const size_t smem = permute_block_smem(E);
    *nlaunch += 1;
    return launch_pdl(permute_single_block_kernel, dim3(1), dim3(kPermBlockTokens), smem, st, idx,
                      T, E, k, counts, offsets, perm, inv, status, touched);
  }
  cudaError_t err = launch_pdl(permute_count_kernel, dim3(nblk), dim3(kPermBlockTokens),
                               E * sizeof(int), st, idx, T, E, k, blk_base, status);
  if (err != cudaSuccess) return err;
  err = launch_pdl(permute_scan_kernel, dim3(1), dim3(1024), 0, st, blk_base, nblk, E, counts,
                   offsets, touched);
  if (err != cudaSuccess) return err;
  *nlaunch += 3;
  return launch_pdl(permute_scatter_kernel, dim3(nblk), dim3(kPermBlockTokens),
                    E * kWordsPerBlock * sizeof(unsigned), st, idx, T, E, k,
                    static_cast<const int32_t*>(blk_base), perm, inv, status);
}

// xperm[r] = h[perm[r]] for every grouped row r (16-byte vector copies).  A
// token id outside [0, T) (left by an invalid routing) yields a zero row.
// One warp per row, the grid's warps striding over the rows; each lane keeps
// eight 16-byte loads in flight before it stores them.
constexpr int kGatherThreads = 256;
constexpr int kGatherUnroll = 8;

__global__ void __launch_bounds__(kGatherThreads) gather_rows_kernel(
    const uint16_t* __restrict__ h, const int32_t* __restrict__ perm, int rows, int D, int T,
    uint16_t* __restrict__ xperm, int* __restrict__ counters, int ncounters) {
  ptx::pdl_launch_dependents();
  ptx::pdl_wait();
  if (blockIdx.x == 0)
    for (int i = threadIdx.x; i < ncounters; i += blockDim.x) counters[i] = 0;
  const int lane = threadIdx.x & 31;
  const int wpb = kGatherThreads / 32;
  const int nwarps = gridDim.x * wpb;
  const int n16 = D / 8;
  for (int r = blockIdx.x * wpb + (threadIdx.x >> 5); r < rows; r += nwarps) {
    const int t = perm[r];
    uint4* dst = reinterpret_cast<uint4*>(xperm + (size_t)r * D);
    if (t < 0 || t >= T) {
      for (int i = lane; i < n16; i += 32) dst[i] = make_uint4(0, 0, 0, 0);
      continue;
    }
    const uint4* src = reinterpret_cast<const uint4*>(h + (size_t)t * D);
    for (int i0 = lane; i0 < n16; i0 += 32 * kGatherUnroll) {
      uint4 v[kGatherUnroll];
#pragma unroll
      for (int u = 0; u < kGatherUnroll; ++u)
        if (i0 + 32 * u < n16) v[u] = src[i0 + 32 * u];
#pragma unroll
      for (int u = 0; u < kGatherUnroll; ++u)
        if (i0 + 32 * u < n16) dst[i0 + 32 * u] = v[u];
    }
  }
}

cudaError_t launch_gather_rows(const uint16_t* h, const int32_t* perm, int rows, int D, int T,
                               uint16_t* xperm, int* counters, int ncounters, cudaStream_t st) {
  if (rows == 0) return cudaSuccess;
  const int wpb = kGatherThreads / 32;
  int blocks = (rows + wpb - 1) / wpb;
  const int cap = num_sms() * 4;
  if (blocks > cap) blocks = cap;
  return launch_pdl(gather_rows_kernel, dim3(blocks), dim3(kGatherThreads), 0, st, h, perm, rows,
                    D, T, xperm, counters, ncounters);
}

}  // namespace moe
