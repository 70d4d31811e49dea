// CUDA-core (SIMT) kernels: the fp32 instance of the indexer and of the
// sparse attention, plus attention shapes that the tensor-core kernel does
// not take.  Exact fp32 FMA arithmetic; no tensor cores.
//
// DeepSeek-V3.2 model doc (Transformers), section "DeepSeek Sparse Attention
// (DSA)": item 1 (index scores of each query against all previous keys) and
// item 2 (attention over the selected tokens only).
#include "dsa_common.cuh"
#include "dsa_internal.h"

namespace dsa {
namespace {

// ------------------------------------------------------------- indexer --
// grid (ceil(s_max/128), n_q, B), 128 threads: one thread per key.
template <typename T>
__global__ void __launch_bounds__(128) indexer_simt_kernel(const T* __restrict__ q, const T* __restrict__ k,
                                                           const float* __restrict__ w,
                                                           const int32_t* __restrict__ ctx_len,
                                                           const int32_t* __restrict__ q_pos0, int t_off,
                                                           float* __restrict__ scores, int64_t ld, int n_q,
                                                           int s_max, int H, int D, float scale) {
  extern __shared__ float sm[];  // q row [H*D], w row [H]
  const int b = blockIdx.z, t = blockIdx.y;
  const int64_t qrow = static_cast<int64_t>(b) * n_q + t;
  for (int i = threadIdx.x; i < H * D; i += blockDim.x) sm[i] = to_f32(q[qrow * H * D + i]);
  for (int i = threadIdx.x; i < H; i += blockDim.x) sm[H * D + i] = w[qrow * H + i];
  __syncthreads();
  const int L = min(max(ctx_len[b], 0), s_max);
  const int p = q_pos0[b] + t_off + t;
  const int s = blockIdx.x * 128 + threadIdx.x;
  if (s >= L) return;
  float res = -INFINITY;
  if (s <= p) {
    const T* kr = k + (static_cast<int64_t>(b) * s_max + s) * D;
    float acc = 0.f;
    for (int h = 0; h < H; ++h) {
      float dot = 0.f;
      for (int d = 0; d < D; ++d) dot = fmaf(sm[h * D + d], to_f32(kr[d]), dot);
      acc = fmaf(sm[H * D + h], fmaxf(scale * dot, 0.f), acc);
    }
    res = acc;
  }
  scores[qrow * ld + s] = res;
}

// ----------------------------------------------------------- attention --
// One warp per (query, head); lanes split the feature dimensions.  Online
// softmax in base 2 with the logit scale folded into q.
template <typename T, int DQ, int DV>
__global__ void __launch_bounds__(256) attn_simt_kernel(const T* __restrict__ q, const T* __restrict__ kv,
                                                        const T* __restrict__ v, const int32_t* __restrict__ idx,
                                                        const int32_t* __restrict__ ctx_len, T* __restrict__ out,
                                                        float* __restrict__ lse, int n_q, int s_max, int H,
                                                        int KVH, int k, float sm_scale, uint32_t* err) {
  constexpr int d_qk = DQ * 32, d_v = DV * 32;
  const int r = blockIdx.x;
  const int b = r / n_q;
  const int h = blockIdx.y * blockDim.y + threadIdx.y;
  if (h >= H) return;
  const int g = h / (H / KVH);
  const int lane = threadIdx.x;
  const int L = min(max(ctx_len[b], 0), s_max);
  const float qs = sm_scale * 1.4426950408889634f;  // log2(e)
  float qr[DQ];
  const T* qp = q + (static_cast<int64_t>(r) * H + h) * d_qk;
#pragma unroll
  for (int i = 0; i < DQ; ++i) qr[i] = to_f32(qp[lane + 32 * i]) * qs;
  float m = -INFINITY, l = 0.f;
  float o[DV];
#pragma unroll
  for (int i = 0; i < DV; ++i) o[i] = 0.f;
  const int32_t* sel = idx + static_cast<int64_t>(r) * k;
  bool bad = false;
  for (int j = 0; j < k; ++j) {
    const int s = __ldg(sel + j);
    if (s < 0) continue;
    if (s >= L) { bad = true; continue; }
    const T* kr = kv + ((static_cast<int64_t>(b) * s_max + s) * KVH + g) * d_qk;
    float dot = 0.f;
#pragma unroll
    for (int i = 0; i < DQ; ++i) dot = fmaf(qr[i], to_f32(kr[lane + 32 * i]), dot);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, off);
    const float mn = fmaxf(m, dot);
    const float corr = exp2f(m - mn);
    const float pj = exp2f(dot - mn);
    l = fmaf(l, corr, pj);
    const T* vr = v ? v + ((static_cast<int64_t>(b) * s_max + s) * KVH + g) * d_v : kr;
#pragma unroll
    for (int i = 0; i < DV; ++i) o[i] = fmaf(o[i], corr, pj * to_f32(vr[lane + 32 * i]));
    m = mn;
  }
  if (bad && lane == 0) raise_error(err, kErrBadIndex);
  const float inv = l > 0.f ? 1.f / l : 0.f;
  T* op = out + (static_cast<int64_t>(r) * H + h) * d_v;
#pragma unroll
  for (int i = 0; i < DV; ++i) op[lane + 32 * i] = from_f32<T>(o[i] * inv);
  if (lse != nullptr && lane == 0)
    lse[static_cast<int64_t>(r) * H + h] = l > 0.f ? (m + log2f(l)) * 0.6931471805599453f : -INFINITY;
}

template <typename T, int DQ, int DV>
void launch_attn_simt(const AttnArgs& a) {
  const int hpb = std::min(8, a.H);
  dim3 block(32, hpb);
  dim3 grid(a.B * a.n_q, (a.H + hpb - 1) / hpb);
  attn_simt_kernel<T, DQ, DV><<<grid, block, 0, a.stream>>>(
      static_cast<const T*>(a.q), static_cast<const T*>(a.kv), static_cast<const T*>(a.v), a.idx, a.ctx_len,
      static_cast<T*>(a.out), a.lse, a.n_q, a.s_max, a.H, a.KVH, a.k, a.sm_scale, a.err);
}

template <typename T>
dsa_status_t dispatch_attn_simt(const AttnArgs& a) {
  if (a.d_qk == 32 && a.d_v == 32) launch_attn_simt<T, 1, 1>(a);
  else if (a.d_qk == 64 && a.d_v == 64) launch_attn_simt<T, 2, 2>(a);
  else if (a.d_qk == 128 && a.d_v == 128) launch_attn_simt<T, 4, 4>(a);
  else if (a.d_qk == 576 && a.d_v == 512) launch_attn_simt<T, 18, 16>(a);
  else return DSA_ERR_UNSUPPORTED;
  return cudaGetLastError() == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

}  // namespace

dsa_status_t indexer_simt(const IndexerArgs& a) {
  if (a.D > 256 || a.H > 128) return DSA_ERR_UNSUPPORTED;
  const size_t smem = static_cast<size_t>(a.H * a.D + a.H) * sizeof(float);
  dim3 grid((a.s_max + 127) / 128, a.n_q, a.B);
  if (a.dtype == DSA_F32) {
    if (smem > 48 * 1024 &&
        cudaFuncSetAttribute(indexer_simt_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem)) != cudaSuccess)
      return DSA_ERR_CUDA;
    indexer_simt_kernel<float><<<grid, 128, smem, a.stream>>>(
        static_cast<const float*>(a.q_idx), static_cast<const float*>(a.k_idx), a.w, a.ctx_len, a.q_pos0, a.t_off,
        a.scores, a.ld, a.n_q, a.s_max, a.H, a.D, a.idx_scale);
  } else {
    return DSA_ERR_UNSUPPORTED;
  }
  return cudaGetLastError() == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

dsa_status_t attn_simt(const AttnArgs& a) {
  if (a.KVH < 1 || a.H % a.KVH != 0) return DSA_ERR_UNSUPPORTED;
  if (a.dtype == DSA_F32) return dispatch_attn_simt<float>(a);
  if (a.dtype == DSA_BF16) return dispatch_attn_simt<__nv_bfloat16>(a);
  return DSA_ERR_UNSUPPORTED;
}

}  // namespace dsa
