// Warp-level Hadamard rotation + FP8 (E4M3) quantisation of one 128-element
// row, shared by the query quantiser and the cache append.
//
// DeepSeek-V3.2 model doc (Transformers), section "DeepSeek Sparse Attention
// (DSA)", item 1: the reference indexer runs in FP8 after the orthogonal
// Hadamard transform `rotate_activation` (Hq.Hk = q.k).  Here: y = H x with
// the orthonormal 128-point Sylvester-Hadamard matrix, one scale per row
// sigma = max|y| / 448 (1 for an all-zero row), codes e4m3(y / sigma) rounded
// to nearest even with saturation.
//
// Lane l holds elements 4l..4l+3.  The fast transform is the butterfly
// network: strides 1 and 2 inside a lane, 4..64 across lanes with shuffles.
#pragma once

#include <cuda_fp8.h>

#include "dsa_common.cuh"

namespace dsa {

// v: this lane's 4 elements in; returns the lane's 4 codes packed (element
// 4l + c in byte c) and the row's scale in *sigma (same in every lane).
__device__ __forceinline__ uint32_t rotate_quant_e4m3(float v[4], float* sigma) {
  const int lane = lane_id();
  {
    // strides 1 and 2 (inside the lane)
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
  const float s = amax > 0.f ? __fdiv_rn(amax, 448.f) : 1.f;
  const __nv_fp8x2_storage_t lo =
      __nv_cvt_float2_to_fp8x2(make_float2(__fdiv_rn(v[0], s), __fdiv_rn(v[1], s)), __NV_SATFINITE, __NV_E4M3);
  const __nv_fp8x2_storage_t hi =
      __nv_cvt_float2_to_fp8x2(make_float2(__fdiv_rn(v[2], s), __fdiv_rn(v[3], s)), __NV_SATFINITE, __NV_E4M3);
  *sigma = s;
  return static_cast<uint32_t>(lo) | (static_cast<uint32_t>(hi) << 16);
}

}  // namespace dsa
