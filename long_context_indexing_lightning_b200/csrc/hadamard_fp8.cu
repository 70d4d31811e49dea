// Hadamard rotation + FP8 (E4M3) quantisation of 128-element rows (the
// arithmetic is in fp8_rows.cuh).  One warp per row, HBM-bound: reads 2 (or
// 4) bytes and writes 1 byte per element plus 4 bytes of scale per row.
#include "dsa_common.cuh"
#include "dsa_internal.h"
#include "fp8_rows.cuh"

namespace dsa {
namespace {

constexpr int kDim = 128;

template <typename T>
__global__ void __launch_bounds__(256) hadamard_quant_kernel(const T* __restrict__ x, int64_t rows,
                                                             uint8_t* __restrict__ x8, float* __restrict__ scale) {
  const int64_t r = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  if (r >= rows) return;  // whole warps leave together (rows are warp-granular)
  const int lane = lane_id();
  float v[4];
  const T* xr = x + r * kDim + 4 * lane;
#pragma unroll
  for (int c = 0; c < 4; ++c) v[c] = to_f32(xr[c]);
  float sigma;
  const uint32_t packed = rotate_quant_e4m3(v, &sigma);
  *reinterpret_cast<uint32_t*>(x8 + r * kDim + 4 * lane) = packed;
  if (lane == 0) scale[r] = sigma;
}

}  // namespace

dsa_status_t hadamard_quant(const void* x, int x_dtype, int64_t rows, int dim, uint8_t* x8, float* scale,
                            cudaStream_t stream) {
  if (dim != kDim) return DSA_ERR_UNSUPPORTED;
  if (rows == 0) return DSA_OK;
  const int64_t threads = rows * 32;
  const int64_t blocks = (threads + 255) / 256;
  if (blocks > INT32_MAX) return DSA_ERR_UNSUPPORTED;
  if (x_dtype == DSA_BF16)
    hadamard_quant_kernel<__nv_bfloat16><<<static_cast<unsigned>(blocks), 256, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(x), rows, x8, scale);
  else if (x_dtype == DSA_F32)
    hadamard_quant_kernel<float><<<static_cast<unsigned>(blocks), 256, 0, stream>>>(static_cast<const float*>(x),
                                                                                   rows, x8, scale);
  else
    return DSA_ERR_UNSUPPORTED;
  return cudaGetLastError() == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

}  // namespace dsa
