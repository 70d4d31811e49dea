// Cache append: each new token's index key and attention rows written at its
// sequence position, before the step scores them.
//
// DeepSeek-V3.2 model doc (Transformers), section "DeepSeek Sparse Attention
// (DSA)": the indexer keeps its own small per-token key cache (single head,
// index_head_dim wide) beside the main K/V cache, updated through
// update_indexer(); the reference indexer runs in FP8 after the Hadamard
// rotation (item 1).
//
// One warp per new token (b, i), written to cache row pos[b] + i:
//   * index key: copied (F32 / BF16 cache), or rotated by the 128-point
//     Hadamard and quantised to e4m3 with one scale per row (E4M3 cache; the
//     arithmetic of fp8_rows.cuh, the same as the query quantiser's),
//   * attention rows: the kv row (kv_heads x d_qk) and, in the separate-V
//     form, the v row (kv_heads x d_v), copied 16 bytes a lane.
// HBM-bound.  Rows outside [0, s_max) are skipped and set kErrBadIndex.
#include "dsa_common.cuh"
#include "dsa_internal.h"
#include "fp8_rows.cuh"

namespace dsa {
namespace {

constexpr int kThreadsPerBlock = 256;

// Warp copy of `bytes` (a multiple of 4): 16-byte chunks when both ends and
// the size allow, else 4-byte words.  Each lane issues all of its loads of a
// 2 KB span (16-byte case) before its stores, so a warp keeps several
// requests in flight instead of one.
__device__ __forceinline__ void warp_copy(char* dst, const char* src, int64_t bytes, int lane) {
  if (((reinterpret_cast<uintptr_t>(dst) | reinterpret_cast<uintptr_t>(src) | static_cast<uintptr_t>(bytes)) & 15u) ==
      0) {
    constexpr int kU = 4;  // chunks per lane per span: 4 x 32 x 16 B = 2 KB
    for (int64_t base = 0; base < bytes; base += kU * 32 * 16) {
      uint4 v[kU];
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const int64_t o = base + (u * 32 + lane) * 16;
        if (o < bytes) v[u] = __ldg(reinterpret_cast<const uint4*>(src + o));
      }
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const int64_t o = base + (u * 32 + lane) * 16;
        if (o < bytes) *reinterpret_cast<uint4*>(dst + o) = v[u];
      }
    }
  } else {
    for (int64_t o = lane * 4; o < bytes; o += 32 * 4)
      *reinterpret_cast<uint32_t*>(dst + o) = __ldg(reinterpret_cast<const uint32_t*>(src + o));
  }
}

template <bool kFP8, typename TK>
__global__ void __launch_bounds__(kThreadsPerBlock) cache_append_kernel(AppendArgs P) {
  pdl_wait();
  const int64_t tok = (static_cast<int64_t>(blockIdx.x) * kThreadsPerBlock + threadIdx.x) >> 5;
  if (tok >= static_cast<int64_t>(P.B) * P.n_new) return;  // whole warps leave together
  const int lane = lane_id();
  const int b = static_cast<int>(tok / P.n_new), i = static_cast<int>(tok % P.n_new);
  const int64_t row = static_cast<int64_t>(__ldg(P.pos + b)) + i;
  if (row < 0 || row >= P.s_max) {
    if (lane == 0) raise_error(P.err, kErrBadIndex);
    return;
  }
  const int64_t dst = static_cast<int64_t>(b) * P.s_max + row;
  // All of this lane's loads first (the latent row in up to 4 x 16 bytes, the
  // key part), then the key's rotation, then the stores: every request of the
  // warp is in flight at once.  Rows over 2 KB, unaligned rows and the
  // separate-V form take the general copy.
  const char* kvs = static_cast<const char*>(P.kv_new) + tok * P.kv_row_bytes;
  char* kvd = static_cast<char*>(P.kv_cache) + dst * P.kv_row_bytes;
  const bool kv_fast = P.v_new == nullptr && P.kv_row_bytes <= 4 * 32 * 16 &&
                       ((reinterpret_cast<uintptr_t>(kvs) | reinterpret_cast<uintptr_t>(kvd) |
                         static_cast<uintptr_t>(P.kv_row_bytes)) & 15u) == 0;
  uint4 kvr[4];
  if (kv_fast) {
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int64_t o = (u * 32 + lane) * 16;
      if (o < P.kv_row_bytes) kvr[u] = __ldg(reinterpret_cast<const uint4*>(kvs + o));
    }
  }
  char* kdst = static_cast<char*>(P.k_cache) + dst * P.k_row_bytes;
  const char* ksrc = static_cast<const char*>(P.k_new) + tok * (kFP8 ? 128 * sizeof(TK) : P.k_row_bytes);
  const bool key16 = !kFP8 && P.k_row_bytes <= 32 * 16 &&
                     ((reinterpret_cast<uintptr_t>(kdst) | reinterpret_cast<uintptr_t>(ksrc) |
                       static_cast<uintptr_t>(P.k_row_bytes)) & 15u) == 0;
  float kv4[4];
  uint4 kchunk = make_uint4(0u, 0u, 0u, 0u);
  if (kFP8) {
    const TK* kr = reinterpret_cast<const TK*>(ksrc) + 4 * lane;
#pragma unroll
    for (int c = 0; c < 4; ++c) kv4[c] = to_f32(kr[c]);
  } else if (key16 && lane * 16 < P.k_row_bytes) {
    kchunk = __ldg(reinterpret_cast<const uint4*>(ksrc + lane * 16));
  }
  if (!kv_fast) {
    warp_copy(kvd, kvs, P.kv_row_bytes, lane);
    if (P.v_new != nullptr)
      warp_copy(static_cast<char*>(P.v_cache) + dst * P.v_row_bytes,
                static_cast<const char*>(P.v_new) + tok * P.v_row_bytes, P.v_row_bytes, lane);
  }
  uint32_t packed = 0;
  float sigma = 0.f;
  if (kFP8) packed = rotate_quant_e4m3(kv4, &sigma);
  if (kv_fast) {
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int64_t o = (u * 32 + lane) * 16;
      if (o < P.kv_row_bytes) *reinterpret_cast<uint4*>(kvd + o) = kvr[u];
    }
  }
  if (kFP8) {
    reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(P.k_cache) + dst * 128)[lane] = packed;
    if (lane == 0) P.k_scale[dst] = sigma;
  } else if (key16) {
    if (lane * 16 < P.k_row_bytes) *reinterpret_cast<uint4*>(kdst + lane * 16) = kchunk;
  } else {
    warp_copy(kdst, ksrc, P.k_row_bytes, lane);
  }
}

}  // namespace

dsa_status_t cache_append(const AppendArgs& a, bool fp8, int k_new_dtype, cudaStream_t stream) {
  const int64_t toks = static_cast<int64_t>(a.B) * a.n_new;
  if (toks == 0) return DSA_OK;
  const int64_t blocks = (toks * 32 + kThreadsPerBlock - 1) / kThreadsPerBlock;
  if (blocks > INT32_MAX) return DSA_ERR_UNSUPPORTED;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(blocks), 1, 1);
  cfg.blockDim = dim3(kThreadsPerBlock, 1, 1);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1] = {pdl_attribute()};
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e;
  if (!fp8)
    e = cudaLaunchKernelEx(&cfg, cache_append_kernel<false, float>, a);
  else if (k_new_dtype == DSA_BF16)
    e = cudaLaunchKernelEx(&cfg, cache_append_kernel<true, __nv_bfloat16>, a);
  else if (k_new_dtype == DSA_F32)
    e = cudaLaunchKernelEx(&cfg, cache_append_kernel<true, float>, a);
  else
    return DSA_ERR_UNSUPPORTED;
  return e == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

}  // namespace dsa
