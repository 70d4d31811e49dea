// Hadamard rotation + FP8 (E4M3) quantisation of 128-element rows.
//
// DeepSeek-V3.2 model doc (Transformers), section "DeepSeek Sparse Attention
// (DSA)", item 1: the reference indexer runs in FP8 after the orthogonal
// Hadamard transform `rotate_activation` (Hq.Hk = q.k).  Here: y = H x with
// the orthonormal 128-point Sylvester-Hadamard matrix, one scale per row
// sigma = max|y| / 448, codes e4m3(y / sigma) rounded to nearest even with
// saturation.
//
// One warp per row; lane l holds elements 4l..4l+3.  The fast transform is
// the butterfly network: strides 1 and 2 inside a lane, 4..64 across lanes
// with shuffles.  HBM-bound: reads 2 (or 4) bytes and writes 1 byte per
// element plus 4 bytes of scale per row.
#include <cuda_fp8.h>

#include "dsa_common.cuh"
#include "dsa_internal.h"

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
  // stride 1 and 2 (inside the lane)
  {
    const float a0 = v[0] + v[1], a1 = v[0] - v[1], a2 = v[2] + v[3], a3 = v[2] - v[3];
    v[0] = a0 + a2;
    v[1] = a1 + a3;
    v[2] = a0 - a2;
    v[3] = a1 - a3;
  }
  // strides 4 .. 64 (lane masks 1 .. 16)
#pragma unroll
  for (int m = 1; m < 32; m <<= 1) {
    const bool upper = (lane & m) != 0;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const float o = __shfl_xor_sync(0xffffffffu, v[c], m);
      v[c] = upper ? (o - v[c]) : (v[c] + o);
    }
  }
  const float inv_sqrt = 0.08838834764831845f;  // 1/sqrt(128)
  float amax = 0.f;
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    v[c] *= inv_sqrt;
    amax = fmaxf(amax, fabsf(v[c]));
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
  const float sigma = amax > 0.f ? __fdiv_rn(amax, 448.f) : 1.f;
  const __nv_fp8x2_storage_t lo =
      __nv_cvt_float2_to_fp8x2(make_float2(__fdiv_rn(v[0], sigma), __fdiv_rn(v[1], sigma)), __NV_SATFINITE, __NV_E4M3);
  const __nv_fp8x2_storage_t hi =
      __nv_cvt_float2_to_fp8x2(make_float2(__fdiv_rn(v[2], sigma), __fdiv_rn(v[3], sigma)), __NV_SATFINITE, __NV_E4M3);
  const uint32_t packed = static_cast<uint32_t>(lo) | (static_cast<uint32_t>(hi) << 16);
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
