// Grouping of the (token, slot) pairs of one batch of at most
// kPermBlockTokens tokens by a single thread block (blockDim a multiple of 32,
// at most 1024): per-expert counts by shared-memory atomics, an exclusive scan
// over experts, and each pair's rank among the batch's tokens for its expert
// from a per-expert token bitmask (tokens pick distinct experts, so one bit per
// token suffices).  Rows within an expert follow increasing token order, i.e.
// (token, slot) order.  Integer work only: exact and deterministic.  Used by
// the single-block grouping kernel and by the routing kernel's last block.
#pragma once

#include "moe_internal.cuh"

namespace moe {

constexpr int kPermWords = kPermBlockTokens / 32;  // bitmask words per expert

// Dynamic shared memory the block grouping needs.
inline size_t permute_block_smem(int E) {
  return (size_t)E * sizeof(int) + (size_t)E * kPermWords * sizeof(unsigned);
}

// Expert choices of one token read per batch, all loads in flight together.
constexpr int kIdxBatch = 8;
__device__ __forceinline__ void load_idx_batch(const int32_t* row, int j0, int k,
                                               int (&ev)[kIdxBatch]) {
#pragma unroll
  for (int u = 0; u < kIdxBatch; ++u) ev[u] = (j0 + u < k) ? __ldcg(row + j0 + u) : 0;
}

// idx [T, k] is read with L2-coherent loads: it may have been written by
// other blocks of the same grid just before.  Must be called by every thread
// of the block; `sm` is permute_block_smem(E) bytes of shared memory.
__device__ __forceinline__ void permute_block(const int32_t* idx, int T, int E, int k,
                                              int32_t* counts, int32_t* offsets, int32_t* perm,
                                              int32_t* inv, int* status, int32_t* touched,
                                              int* sm) {
  int* cnt = sm;                                           // [E]
  unsigned* mask = reinterpret_cast<unsigned*>(sm + E);    // [E][kPermWords]
  __shared__ int warp_tot[32];
  __shared__ unsigned bad_tok[kPermWords];                 // tokens with an invalid choice
  __shared__ int nz_total;
  const int nthr = blockDim.x;
  for (int i = threadIdx.x; i < E; i += nthr) cnt[i] = 0;
  for (int i = threadIdx.x; i < E * kPermWords; i += nthr) mask[i] = 0u;
  if (threadIdx.x < kPermWords) bad_tok[threadIdx.x] = 0u;
  if (threadIdx.x == 0) nz_total = 0;
  __syncthreads();
  bool any_bad = false;
  for (int t = threadIdx.x; t < T; t += nthr) {
    const int word = t >> 5;
    const unsigned bit = 1u << (t & 31);
    bool bad = false;
    for (int j0 = 0; j0 < k; j0 += kIdxBatch) {
      int ev[kIdxBatch];
      load_idx_batch(idx + (size_t)t * k, j0, k, ev);   // all loads in flight together
#pragma unroll
      for (int u = 0; u < kIdxBatch; ++u) {
        if (j0 + u >= k) break;
        const int e = ev[u];
        if (e < 0 || e >= E) {
          bad = true;
          continue;
        }
        atomicAdd(&cnt[e], 1);
        const unsigned old = atomicOr(&mask[e * kPermWords + word], bit);
        if (old & bit) bad = true;  // the same expert twice in one token
      }
    }
    if (bad) {
      atomicOr(&bad_tok[word], bit);
      any_bad = true;
    }
  }
  __syncthreads();
  // exclusive scan of cnt over experts: thread i owns experts [i*per, (i+1)*per)
  const int per = (E + nthr - 1) / nthr;
  const int e0 = threadIdx.x * per;
  int local = 0;
  for (int e = e0; e < e0 + per && e < E; ++e) local += cnt[e];
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  int incl = local;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += v;
  }
  if (lane == 31) warp_tot[wid] = incl;
  __syncthreads();
  int base = incl - local;
  for (int q = 0; q < wid; ++q) base += warp_tot[q];
  __syncthreads();  // everyone has read warp_tot; cnt becomes the offsets
  int nz = 0;
  for (int e = e0; e < e0 + per && e < E; ++e) {
    const int c = cnt[e];
    counts[e] = c;
    offsets[e] = base;
    cnt[e] = base;
    base += c;
    nz += c > 0;
  }
  if (threadIdx.x == nthr - 1) offsets[E] = base;  // the last thread ends at the total
  if (nz) atomicAdd(&nz_total, nz);
  __syncthreads();
  if (touched && threadIdx.x == 0) *touched = nz_total;
  for (int t = threadIdx.x; t < T; t += nthr) {
    const int word = t >> 5;
    const unsigned bit = 1u << (t & 31);
    if (bad_tok[word] & bit) continue;
    for (int j0 = 0; j0 < k; j0 += kIdxBatch) {
      int ev[kIdxBatch];
      load_idx_batch(idx + (size_t)t * k, j0, k, ev);
#pragma unroll
      for (int u = 0; u < kIdxBatch; ++u) {
        if (j0 + u >= k) break;
        const int e = ev[u];
        const unsigned* m = mask + e * kPermWords;
        int rank = __popc(m[word] & (bit - 1u));
        for (int q = 0; q < word; ++q) rank += __popc(m[q]);
        const int row = cnt[e] + rank;
        perm[row] = t;
        inv[(size_t)t * k + j0 + u] = row;
      }
    }
  }
  if (any_bad && status) atomicOr(status, kStBounds);
}

// Grouping from the per-expert token bitmasks `gmask` [E][kPermWords] that
// the routing blocks filled (bit t of row e: token t chose expert e), by the
// routing kernel's last block.  The counts are the rows' popcounts; the pair
// (t, j) with expert e = idx[t, j] goes to row offsets[e] + (number of tokens
// below t in row e), which is the (token, slot) order of permute_block.  The
// block reads the rows (L2-coherent: other blocks of the grid just set them)
// and clears them for the next call.  Same outputs as permute_block for idx
// rows of distinct in-range experts, which the routing always produces; an
// out-of-range expert raises kStBounds and leaves its pair's perm/inv rows
// unwritten.  Must be called by every thread of the block; `sm` is
// permute_block_smem(E) bytes.
__device__ __forceinline__ void group_from_masks(const int32_t* idx, int T, int E, int k,
                                                 uint32_t* gmask, int32_t* counts,
                                                 int32_t* offsets, int32_t* perm, int32_t* inv,
                                                 int* status, int32_t* touched, int* sm) {
  int* cnt = sm;                                           // [E]
  unsigned* mask = reinterpret_cast<unsigned*>(sm + E);    // [E][W]
  __shared__ int warp_tot[32];
  __shared__ int nz_total;
  const int nthr = blockDim.x;
  const int W = (T + 31) >> 5;                             // words per expert row in use
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  if (threadIdx.x == 0) nz_total = 0;
  // The first batch of pairs' experts is loaded together with the row words
  // (one round trip for both when T * k <= blockDim * kIdxBatch).
  const int npairs = T * k;
  int ev0[kIdxBatch];
#pragma unroll
  for (int u = 0; u < kIdxBatch; ++u) {
    const int pr = u * nthr + threadIdx.x;
    ev0[u] = pr < npairs ? __ldcg(idx + pr) : 0;
  }
  // the row words are loaded in batches with every load in flight before any
  // is stored or cleared
  for (int i0 = 0; i0 < E * W; i0 += nthr * kIdxBatch) {
    uint32_t v[kIdxBatch];
#pragma unroll
    for (int u = 0; u < kIdxBatch; ++u) {
      const int i = i0 + u * nthr + threadIdx.x;
      const int e = i / W, q = i - e * W;
      v[u] = i < E * W ? __ldcg(gmask + (size_t)e * kPermWords + q) : 0u;
    }
#pragma unroll
    for (int u = 0; u < kIdxBatch; ++u) {
      const int i = i0 + u * nthr + threadIdx.x;
      if (i >= E * W) break;
      const int e = i / W, q = i - e * W;
      mask[i] = v[u];
      gmask[(size_t)e * kPermWords + q] = 0u;
    }
  }
  __syncthreads();
  // per-expert counts, then an exclusive scan over experts: thread i owns
  // experts [i*per, (i+1)*per)
  const int per = (E + nthr - 1) / nthr;
  const int e0 = threadIdx.x * per;
  int local = 0;
  for (int e = e0; e < e0 + per && e < E; ++e) {
    int c = 0;
    for (int q = 0; q < W; ++q) c += __popc(mask[e * W + q]);
    cnt[e] = c;
    local += c;
  }
  int incl = local;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += v;
  }
  if (lane == 31) warp_tot[wid] = incl;
  __syncthreads();
  int base = incl - local;
  for (int q = 0; q < wid; ++q) base += warp_tot[q];
  int nz = 0;
  for (int e = e0; e < e0 + per && e < E; ++e) {
    const int c = cnt[e];
    counts[e] = c;
    offsets[e] = base;
    cnt[e] = base;
    base += c;
    nz += c > 0;
  }
  if (threadIdx.x == nthr - 1) offsets[E] = base;  // the last thread ends at the total
  if (nz) atomicAdd(&nz_total, nz);
  __syncthreads();
  if (touched && threadIdx.x == 0) *touched = nz_total;
  // one pair per thread and round: row = offset + rank of t in its expert's row
  bool bad = false;
  for (int p0 = 0; p0 < npairs; p0 += nthr * kIdxBatch) {
    int ev[kIdxBatch];
#pragma unroll
    for (int u = 0; u < kIdxBatch; ++u) {
      const int pr = p0 + u * nthr + threadIdx.x;
      ev[u] = p0 == 0 ? ev0[u] : (pr < npairs ? __ldcg(idx + pr) : 0);
    }
#pragma unroll
    for (int u = 0; u < kIdxBatch; ++u) {
      const int pr = p0 + u * nthr + threadIdx.x;
      if (pr >= npairs) break;
      const int e = ev[u];
      if (e < 0 || e >= E) {
        bad = true;
        continue;
      }
      const int t = pr / k;
      const int word = t >> 5;
      const unsigned* m = mask + e * W;
      int rank = __popc(m[word] & ((1u << (t & 31)) - 1u));
      for (int q = 0; q < word; ++q) rank += __popc(m[q]);
      const int row = cnt[e] + rank;
      perm[row] = t;
      inv[pr] = row;
    }
  }
  if (bad && status) atomicOr(status, kStBounds);
}

}  // namespace moe
