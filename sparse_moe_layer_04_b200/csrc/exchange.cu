// Row gather for the expert-parallel exchange: dst[i] = src[idx[i]] for rows
// of any width that is a multiple of 16 bytes (bf16 token rows before the
// dispatch, fp32 expert-output rows before the return trip).
#include "moe_internal.cuh"
#include "sm100_ptx.cuh"

namespace moe {
namespace {

// One 16-byte vector per thread and step; an index outside [0, src_rows)
// zero-fills its row and raises kStBounds.
__global__ void __launch_bounds__(256) gather_bytes_kernel(const uint4* __restrict__ src,
                                                           int src_rows,
                                                           const int32_t* __restrict__ idx,
                                                           long long n, int row_vecs,
                                                           uint4* __restrict__ dst, int* status) {
  ptx::pdl_launch_dependents();
  ptx::pdl_wait();
  bool bad = false;
  const long long total = n * row_vecs;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total;
       i += (long long)gridDim.x * blockDim.x) {
    const long long r = i / row_vecs;
    const int c = static_cast<int>(i - r * row_vecs);
    const int s = idx[r];
    if (s < 0 || s >= src_rows) {
      bad = true;
      dst[i] = make_uint4(0u, 0u, 0u, 0u);
    } else {
      dst[i] = src[(long long)s * row_vecs + c];
    }
  }
  if (bad && status) atomicOr(status, kStBounds);
}

}  // namespace

cudaError_t launch_gather_bytes(const void* src, int src_rows, const int32_t* idx, int n,
                                int row_bytes, void* dst, int* status, cudaStream_t st) {
  const long long vecs = (long long)n * (row_bytes / 16);
  if (vecs == 0) return cudaSuccess;
  long long blocks = (vecs + 255) / 256;
  const long long cap = 8ll * num_sms();
  if (blocks > cap) blocks = cap;
  return launch_pdl(gather_bytes_kernel, dim3((unsigned)blocks), dim3(256), 0, st,
                    static_cast<const uint4*>(src), src_rows, idx, (long long)n, row_bytes / 16,
                    static_cast<uint4*>(dst), status);
}

}  // namespace moe
