// Stand-alone decoding of FP8 expert weights to bf16 (the same exact decoding
// the FP8 expert-FFN kernel applies on its way into tensor memory).
#include "fp8_convert.cuh"
#include "moe_internal.cuh"
#include "sm100_ptx.cuh"

namespace moe {
namespace {

// One thread per 16 codes of a row: one 16-byte load, two 16-byte stores.
__global__ void __launch_bounds__(256) fp8_dequantize_kernel(const uint8_t* __restrict__ codes,
                                                             const int8_t* __restrict__ exps,
                                                             int R, int K, long long nchunks,
                                                             uint16_t* __restrict__ out,
                                                             int* status) {
  ptx::pdl_launch_dependents();
  ptx::pdl_wait();
  const int cpr = K / 16;                       // chunks per row
  const int RB = (R + fp8::kBlock - 1) / fp8::kBlock;
  const int KB = (K + fp8::kBlock - 1) / fp8::kBlock;
  bool bad = false;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < nchunks;
       i += (long long)gridDim.x * blockDim.x) {
    const long long row = i / cpr;              // row over all groups
    const int kc = static_cast<int>(i - row * cpr) * 16;
    const long long g = row / R;
    const int r = static_cast<int>(row - g * R);
    const int e = exps[(g * RB + r / fp8::kBlock) * KB + kc / fp8::kBlock];
    bad |= !fp8::exp_ok(e);
    const uint32_t s2 = fp8::scale_pair(e);
    const uint4 c = *reinterpret_cast<const uint4*>(codes + i * 16);
    uint4 o0, o1;
    fp8::decode4(c.x, s2, o0.x, o0.y);
    fp8::decode4(c.y, s2, o0.z, o0.w);
    fp8::decode4(c.z, s2, o1.x, o1.y);
    fp8::decode4(c.w, s2, o1.z, o1.w);
    uint4* dst = reinterpret_cast<uint4*>(out + i * 16);
    dst[0] = o0;
    dst[1] = o1;
  }
  if (bad && status) atomicOr(status, kStBounds);
}

}  // namespace

cudaError_t launch_fp8_dequantize(const uint8_t* codes, const int8_t* exps, int G, int R, int K,
                                  uint16_t* out, int* status, cudaStream_t st) {
  const long long nchunks = (long long)G * R * (K / 16);
  if (nchunks == 0) return cudaSuccess;
  long long blocks = (nchunks + 255) / 256;
  const long long cap = 8ll * num_sms();
  if (blocks > cap) blocks = cap;
  return launch_pdl(fp8_dequantize_kernel, dim3((unsigned)blocks), dim3(256), 0, st, codes, exps,
                    R, K, nchunks, out, status);
}

}  // namespace moe
