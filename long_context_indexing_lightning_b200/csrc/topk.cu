// Fine-grained token selection: per query, the index_topk best-scored
// previous keys (DeepSeek-V3.2 model doc, Transformers, section "DeepSeek
// Sparse Attention (DSA)", item 2; index_topk defaults to 2048).
//
// Radix select on order-preserving 32-bit keys, no sort.  One query row is
// split over a thread-block cluster of C CTAs (C = 1..16); each thread keeps
// its PER consecutive keys in registers for the whole selection:
//   * three histogram passes (digits of 11, 11 and 10 bits, most significant
//     first) into shared memory.  Each CTA also totals its histogram in 32
//     groups of 64 bins; through distributed shared memory every CTA sums the
//     C CTAs' group totals, finds the group holding the k-th largest key, then
//     sums only that group's 64 bins over the C CTAs and finds the digit (all
//     CTAs reach the same digit).  After three passes all CTAs know the exact
//     key T of the k-th largest score and how many keys equal to T to keep;
//   * one ordered compaction: per-thread counts of keys > T and == T, a block
//     prefix sum (warp shuffles), CTA totals exchanged across the cluster,
//     then every kept index is written at its final position -- keys > T plus
//     the lowest-indexed keys == T (ties go to the lower index), ascending.
// Rows with at most k candidates are written directly.
#include <cooperative_groups.h>

#include "dsa_common.cuh"
#include "dsa_internal.h"

namespace cg = cooperative_groups;

namespace dsa {
namespace {

constexpr int kBins = 2048;
constexpr int kGroupBins = 64;                    // bins per group total
constexpr int kGroups = kBins / kGroupBins;       // 32
constexpr int kMaxWarps = 32;
constexpr int kMaxCluster = 16;

__device__ __forceinline__ uint32_t warp_incl_scan(uint32_t v) {
  const int lane = lane_id();
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const uint32_t n = __shfl_up_sync(0xffffffffu, v, off);
    if (lane >= off) v += n;
  }
  return v;
}

// Block-wide exclusive scan of one value per thread; the block total goes to
// *total.  Uses `wsum` (kMaxWarps + 1 words).
template <int kThreads>
__device__ __forceinline__ uint32_t block_excl_scan(uint32_t v, uint32_t* wsum, uint32_t* total) {
  constexpr int kWarps = kThreads / 32;
  const int lane = lane_id(), warp = threadIdx.x >> 5;
  const uint32_t incl = warp_incl_scan(v);
  if (lane == 31) wsum[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const uint32_t x = lane < kWarps ? wsum[lane] : 0u;
    const uint32_t xi = warp_incl_scan(x);
    if (lane < kWarps) wsum[lane] = xi - x;
    if (lane == 31) wsum[kWarps] = xi;
  }
  __syncthreads();
  const uint32_t res = wsum[warp] + incl - v;
  *total = wsum[kWarps];
  __syncthreads();
  return res;
}

template <int PER, int kThreads>
__global__ void __launch_bounds__(kThreads, 1024 / kThreads)
    topk_cluster_kernel(const float* __restrict__ scores, int64_t ld, const int32_t* __restrict__ ctx_len,
                        const int32_t* __restrict__ q_pos0, int t_off, int n_q, int s_max, int k,
                        int32_t* __restrict__ idx) {
  pdl_wait();
  __shared__ uint32_t hist[3][kBins];
  __shared__ uint32_t gtot[3][kGroups];   // this CTA's group totals, read by the peers
  __shared__ uint32_t mgroup[kGroups];    // group totals over the cluster
  __shared__ uint32_t mbin[kGroupBins];   // the target group's bins over the cluster
  __shared__ uint32_t s_group, s_gabove;
  __shared__ uint32_t wsum[kMaxWarps + 1];
  __shared__ uint32_t s_digit, s_above;
  __shared__ uint32_t s_tot[2];
  __shared__ uint32_t s_off[2];

  cg::cluster_group cluster = cg::this_cluster();
  const int C = static_cast<int>(cluster.num_blocks());
  const int c = static_cast<int>(cluster.block_rank());
  const int r = blockIdx.x / C;
  const int b = r / n_q, t = r % n_q;
  const int L = min(max(ctx_len[b], 0), s_max);
  const int n = max(0, min(q_pos0[b] + t_off + t + 1, L));  // candidates s in [0, n)
  int32_t* out = idx + static_cast<int64_t>(r) * k;
  const float* row = scores + static_cast<int64_t>(r) * ld;
  const int tid = threadIdx.x;

  if (n <= k) {  // the same for every CTA of the cluster: nobody syncs
    for (int j = c * kThreads + tid; j < k; j += C * kThreads) out[j] = j < n ? j : -1;
    return;
  }

  // this thread's keys: s = s0 .. s0 + PER - 1
  const int s0 = (c * kThreads + tid) * PER;
  uint32_t key[PER];
  uint32_t vmask = 0;
  if (s0 + PER <= n) {
#pragma unroll
    for (int e = 0; e < PER; e += 4) {
      const float4 f = *reinterpret_cast<const float4*>(row + s0 + e);
      key[e] = float_order_key(f.x);
      key[e + 1] = float_order_key(f.y);
      key[e + 2] = float_order_key(f.z);
      key[e + 3] = float_order_key(f.w);
    }
    vmask = (PER == 32) ? 0xffffffffu : ((1u << PER) - 1u);
  } else {
#pragma unroll
    for (int e = 0; e < PER; ++e) {
      const bool v = s0 + e < n;
      key[e] = v ? float_order_key(row[s0 + e]) : 0u;
      vmask |= (v ? 1u : 0u) << e;
    }
  }

  uint32_t prefix = 0, pmask = 0, remaining = static_cast<uint32_t>(k);
#pragma unroll 1
  for (int pass = 0; pass < 3; ++pass) {
    const int shift = pass == 0 ? 21 : (pass == 1 ? 10 : 0);
    const uint32_t dmask = pass == 2 ? 0x3FFu : 0x7FFu;
    for (int i = tid; i < kBins; i += kThreads) hist[pass][i] = 0;
    __syncthreads();
#pragma unroll
    for (int e = 0; e < PER; ++e)
      if (((vmask >> e) & 1u) && (key[e] & pmask) == prefix) atomicAdd(&hist[pass][(key[e] >> shift) & dmask], 1u);
    __syncthreads();
    {
      // group totals: kBins / kThreads consecutive bins a thread, 64 a group
      constexpr int kPerT = kBins / kThreads;
      constexpr int kLanesPerGroup = kGroupBins / kPerT;
      uint32_t v = 0;
#pragma unroll
      for (int q = 0; q < kPerT; ++q) v += hist[pass][tid * kPerT + q];
#pragma unroll
      for (int off = 1; off < kLanesPerGroup; off <<= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
      if ((tid & (kLanesPerGroup - 1)) == 0) gtot[pass][tid / kLanesPerGroup] = v;
    }
    cluster.sync();  // every CTA's histogram and group totals of this pass are complete
    static_assert(kThreads == kGroups * kMaxCluster, "one thread per (group, cluster rank)");
    {
      // sum the C CTAs' group totals: thread = (group, rank), reduced over 16 lanes
      const int g = tid / kMaxCluster, q = tid % kMaxCluster;
      uint32_t v = q < C ? cluster.map_shared_rank(&gtot[pass][0], q)[g] : 0u;
#pragma unroll
      for (int off = 1; off < kMaxCluster; off <<= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
      if (q == 0) mgroup[g] = v;
    }
    __syncthreads();
    if (tid < 32) {
      // the group holding the remaining-th largest key, scanning from the top
      const uint32_t cnt = mgroup[kGroups - 1 - tid];
      const uint32_t incl = warp_incl_scan(cnt);
      if (incl - cnt < remaining && remaining <= incl) {
        s_group = static_cast<uint32_t>(kGroups - 1 - tid);
        s_gabove = incl - cnt;
      }
    }
    __syncthreads();
    const uint32_t G = s_group;
#pragma unroll
    for (int hb = 0; hb < kGroupBins / (kThreads / kMaxCluster); ++hb) {
      // that group's bins summed over the C CTAs: thread = (bin, rank)
      const int bl = hb * (kThreads / kMaxCluster) + tid / kMaxCluster, q = tid % kMaxCluster;
      uint32_t v = q < C ? cluster.map_shared_rank(&hist[pass][0], q)[G * kGroupBins + bl] : 0u;
#pragma unroll
      for (int off = 1; off < kMaxCluster; off <<= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
      if (q == 0) mbin[bl] = v;
    }
    __syncthreads();
    if (tid < 32) {
      // the bin within the group, two bins a lane from the top
      const uint32_t rem = remaining - s_gabove;
      const uint32_t hi = mbin[kGroupBins - 1 - 2 * tid], lo = mbin[kGroupBins - 2 - 2 * tid];
      const uint32_t incl = warp_incl_scan(hi + lo);
      const uint32_t excl = incl - hi - lo;
      if (excl < rem && rem <= incl) {
        if (rem <= excl + hi) {
          s_digit = G * kGroupBins + kGroupBins - 1 - 2 * tid;
          s_above = s_gabove + excl;
        } else {
          s_digit = G * kGroupBins + kGroupBins - 2 - 2 * tid;
          s_above = s_gabove + excl + hi;
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

  pdl_trigger();  // the selection is fixed; only the writes remain
  uint32_t gt = 0, eq = 0;
#pragma unroll
  for (int e = 0; e < PER; ++e) {
    const bool v = (vmask >> e) & 1u;
    gt += (v && key[e] > T) ? 1u : 0u;
    eq += (v && key[e] == T) ? 1u : 0u;
  }
  uint32_t total;
  const uint32_t pre = block_excl_scan<kThreads>((gt << 16) | eq, wsum, &total);
  if (tid == 0) {
    s_tot[0] = total >> 16;
    s_tot[1] = total & 0xFFFFu;
  }
  cluster.sync();  // CTA totals visible across the cluster
  if (tid < 32) {
    // offsets of this CTA: the totals of the lower-ranked CTAs, one remote
    // read per lane, summed across the warp
    uint32_t g = 0, e = 0;
    if (tid < c) {
      const uint32_t* pt = cluster.map_shared_rank(&s_tot[0], tid);
      g = pt[0];
      e = pt[1];
    }
#pragma unroll
    for (int off = 1; off < kMaxCluster; off <<= 1) {
      g += __shfl_xor_sync(0xffffffffu, g, off);
      e += __shfl_xor_sync(0xffffffffu, e, off);
    }
    if (tid == 0) {
      s_off[0] = g;
      s_off[1] = e;
    }
  }
  // every remote read of this CTA is done: arrive now, wait only before
  // leaving (peers may still be reading this CTA's totals), so the index
  // writes below overlap the barrier
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
  __syncthreads();
  const uint32_t gt_off = s_off[0], eq_off = s_off[1];
  uint32_t eq_rank = eq_off + (pre & 0xFFFFu);
  uint32_t pos = gt_off + (pre >> 16) + min(eq_rank, take_eq);
#pragma unroll
  for (int e = 0; e < PER; ++e) {
    if (!((vmask >> e) & 1u)) continue;
    if (key[e] > T) {
      out[pos++] = s0 + e;
    } else if (key[e] == T) {
      if (eq_rank < take_eq) out[pos++] = s0 + e;
      ++eq_rank;
    }
  }
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");  // peers are done with this CTA
}

template <int PER, int kThreads>
dsa_status_t launch_topk(const TopkArgs& a, int C) {
  auto kern = topk_cluster_kernel<PER, kThreads>;
  if (C > 8) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess)
      return DSA_ERR_UNSUPPORTED;
  }
  const int64_t rows = static_cast<int64_t>(a.B) * a.n_q;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(rows * C), 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = a.stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = C;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1] = pdl_attribute();
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, a.scores, a.ld, a.ctx_len, a.q_pos0, a.t_off, a.n_q, a.s_max,
                                           a.k, a.idx);
  return e == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

}  // namespace

size_t topk_workspace_bytes(int, int, int, int) { return 0; }

dsa_status_t topk_radix(const TopkArgs& a) {
  const int64_t rows = static_cast<int64_t>(a.B) * a.n_q;
  if (rows == 0) return DSA_OK;
  const int num_sms = std::max(1, device_sm_count(a.device));
  const int64_t n_max = std::max(1, a.s_max);
  // 512 threads x 32 keys (16K keys, two CTAs per SM) per cluster rank; when
  // a handful of long rows would leave SMs idle, 8 keys a thread instead
  // (more CTAs per row); at most 16 CTAs per row.
  constexpr int kT = 512;
  int per = 32;
  if (rows * ((n_max + 32 * kT - 1) / (32 * kT)) < 2 * num_sms && (n_max + 8 * kT - 1) / (8 * kT) <= 8) per = 8;
  const int64_t C = (n_max + static_cast<int64_t>(per) * kT - 1) / (static_cast<int64_t>(per) * kT);
  if (C > kMaxCluster) return DSA_ERR_UNSUPPORTED;
  if (rows * C > INT32_MAX) return DSA_ERR_UNSUPPORTED;
  return per == 8 ? launch_topk<8, kT>(a, static_cast<int>(C)) : launch_topk<32, kT>(a, static_cast<int>(C));
}

}  // namespace dsa
