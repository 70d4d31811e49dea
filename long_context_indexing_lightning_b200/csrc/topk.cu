// Fine-grained token selection: per query, the index_topk best-scored
// previous keys (DeepSeek-V3.2 model doc, Transformers, section "DeepSeek
// Sparse Attention (DSA)", item 2; index_topk defaults to 2048).
//
// Radix select on order-preserving 32-bit keys, no sort:
//   * three histogram passes over the candidate row (digits of 11, 11 and
//     10 bits, most significant first) in shared memory find the exact key T
//     of the k-th largest score and how many keys equal to T to keep;
//   * one ordered compaction pass keeps every key > T and the lowest-indexed
//     keys == T (ties go to the lower index), emitting indices in ascending
//     order.  Per-thread segment counts are combined with warp shuffles and a
//     block prefix sum, so the output is deterministic.
// One 1024-thread CTA per query row; rows with at most k candidates are
// written directly.
#include "dsa_common.cuh"
#include "dsa_internal.h"

namespace dsa {
namespace {

constexpr int kThreads = 1024;
constexpr int kWarps = kThreads / 32;
constexpr int kBins = 2048;
constexpr int kSeg = 8;  // consecutive elements per thread in the compaction pass

__device__ __forceinline__ uint32_t warp_incl_scan(uint32_t v) {
  const int lane = lane_id();
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const uint32_t n = __shfl_up_sync(0xffffffffu, v, off);
    if (lane >= off) v += n;
  }
  return v;
}

// Block-wide exclusive scan of one value per thread; returns the exclusive
// prefix and writes the block total to *total.  Uses `wsum` (kWarps words).
__device__ __forceinline__ uint32_t block_excl_scan(uint32_t v, uint32_t* wsum, uint32_t* total) {
  const int lane = lane_id(), warp = threadIdx.x >> 5;
  const uint32_t incl = warp_incl_scan(v);
  if (lane == 31) wsum[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const uint32_t x = wsum[lane];
    const uint32_t xi = warp_incl_scan(x);
    wsum[lane] = xi - x;
    if (lane == 31) wsum[kWarps] = xi;
  }
  __syncthreads();
  const uint32_t res = wsum[warp] + incl - v;
  *total = wsum[kWarps];
  __syncthreads();
  return res;
}

__global__ void __launch_bounds__(kThreads) topk_radix_kernel(const float* __restrict__ scores, int64_t ld,
                                                              const int32_t* __restrict__ ctx_len,
                                                              const int32_t* __restrict__ q_pos0, int t_off,
                                                              int n_q, int s_max, int k, int32_t* __restrict__ idx) {
  __shared__ uint32_t hist[kBins];
  __shared__ uint32_t wsum[kWarps + 1];
  __shared__ uint32_t s_digit, s_above;

  const int r = blockIdx.x;
  const int b = r / n_q, t = r % n_q;
  const int L = min(max(ctx_len[b], 0), s_max);
  const int n = max(0, min(q_pos0[b] + t_off + t + 1, L));  // candidates s in [0, n)
  int32_t* out = idx + static_cast<int64_t>(r) * k;
  const float* row = scores + static_cast<int64_t>(r) * ld;
  const int tid = threadIdx.x;

  if (n <= k) {
    for (int j = tid; j < k; j += kThreads) out[j] = j < n ? j : -1;
    return;
  }

  uint32_t prefix = 0, pmask = 0, remaining = static_cast<uint32_t>(k);
#pragma unroll 1
  for (int pass = 0; pass < 3; ++pass) {
    const int shift = pass == 0 ? 21 : (pass == 1 ? 10 : 0);
    const uint32_t dmask = pass == 2 ? 0x3FFu : 0x7FFu;
    for (int i = tid; i < kBins; i += kThreads) hist[i] = 0;
    __syncthreads();
    const int n4 = n >> 2;
    const float4* row4 = reinterpret_cast<const float4*>(row);
    for (int i = tid; i < n4; i += kThreads) {
      const float4 f = row4[i];
      const uint32_t u0 = float_order_key(f.x), u1 = float_order_key(f.y);
      const uint32_t u2 = float_order_key(f.z), u3 = float_order_key(f.w);
      if ((u0 & pmask) == prefix) atomicAdd(&hist[(u0 >> shift) & dmask], 1u);
      if ((u1 & pmask) == prefix) atomicAdd(&hist[(u1 >> shift) & dmask], 1u);
      if ((u2 & pmask) == prefix) atomicAdd(&hist[(u2 >> shift) & dmask], 1u);
      if ((u3 & pmask) == prefix) atomicAdd(&hist[(u3 >> shift) & dmask], 1u);
    }
    for (int s = (n4 << 2) + tid; s < n; s += kThreads) {
      const uint32_t u = float_order_key(row[s]);
      if ((u & pmask) == prefix) atomicAdd(&hist[(u >> shift) & dmask], 1u);
    }
    __syncthreads();
    // Digit holding the remaining-th largest key: scan bins from the top.
    if (tid < 32) {
      const int lane = tid;
      constexpr int kPer = kBins / 32;
      const int top = kBins - 1 - lane * kPer;  // this lane scans bins top .. top-kPer+1
      uint32_t local = 0;
      for (int i = 0; i < kPer; ++i) local += hist[top - i];
      const uint32_t incl = warp_incl_scan(local);
      const uint32_t excl = incl - local;
      if (excl < remaining && remaining <= incl) {
        uint32_t cum = excl;
        for (int i = 0; i < kPer; ++i) {
          const uint32_t c = hist[top - i];
          if (cum + c >= remaining) {
            s_digit = static_cast<uint32_t>(top - i);
            s_above = cum;
            break;
          }
          cum += c;
        }
      }
    }
    __syncthreads();
    prefix |= s_digit << shift;
    pmask |= dmask << shift;
    remaining -= s_above;
    __syncthreads();
  }
  const uint32_t T = prefix;
  const uint32_t take_eq = remaining;  // keys == T to keep, lowest index first

  // Ordered compaction: thread `tid` owns elements [base + tid*kSeg, +kSeg).
  uint32_t gt_done = 0, eq_done = 0;
  for (int base = 0; base < n; base += kThreads * kSeg) {
    const int s0 = base + tid * kSeg;
    uint32_t keys[kSeg];
#pragma unroll
    for (int e = 0; e < kSeg; ++e) {
      const int s = s0 + e;
      keys[e] = (s < n) ? float_order_key(row[s]) : 0u;  // 0 is below every real key
    }
    uint32_t gt = 0, eq = 0;
#pragma unroll
    for (int e = 0; e < kSeg; ++e) {
      gt += keys[e] > T;
      eq += (s0 + e < n) && keys[e] == T;
    }
    uint32_t total;
    const uint32_t pre = block_excl_scan((gt << 16) | eq, wsum, &total);
    const uint32_t gt_before = gt_done + (pre >> 16);
    uint32_t eq_rank = eq_done + (pre & 0xFFFFu);
    uint32_t pos = gt_before + min(eq_rank, take_eq);
#pragma unroll
    for (int e = 0; e < kSeg; ++e) {
      const int s = s0 + e;
      if (s >= n) break;
      if (keys[e] > T) {
        out[pos++] = s;
      } else if (keys[e] == T) {
        if (eq_rank < take_eq) out[pos++] = s;
        ++eq_rank;
      }
    }
    gt_done += total >> 16;
    eq_done += total & 0xFFFFu;
  }
}

}  // namespace

size_t topk_workspace_bytes(int, int, int, int) { return 0; }

dsa_status_t topk_radix(const TopkArgs& a) {
  const int64_t rows = static_cast<int64_t>(a.B) * a.n_q;
  if (rows == 0) return DSA_OK;
  if (rows > INT32_MAX) return DSA_ERR_UNSUPPORTED;
  topk_radix_kernel<<<static_cast<unsigned>(rows), kThreads, 0, a.stream>>>(
      a.scores, a.ld, a.ctx_len, a.q_pos0, a.t_off, a.n_q, a.s_max, a.k, a.idx);
  return cudaGetLastError() == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

}  // namespace dsa
