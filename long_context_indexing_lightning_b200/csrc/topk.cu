// Fine-grained token selection: per query, the index_topk best-scored
// previous keys (DeepSeek-V3.2 model doc, Transformers, section "DeepSeek
// Sparse Attention (DSA)", item 2; index_topk defaults to 2048).
//
// Radix select on order-preserving 32-bit keys, no sort.  One query row is
// split over a thread-block cluster of C CTAs (C = 1..16, 16K keys a CTA in
// two chunks of 8K, read with coalesced loads); when a launch has many rows
// (prefill), C = 1 and each CTA walks its row chunk by chunk.  The key splits into
// digits of 11, 11 and 10 bits; T, the key of the k-th largest score, is
// found digit by digit:
//   1. the first digit's histogram: summed from the partial histograms the
//      indexer's epilogue built (TopkArgs::hist_parts), or counted by each CTA
//      and merged in the cluster's first CTA (the leader); the bin D1 holding
//      the k-th largest key follows;
//   2. each CTA keeps, in index order, its "sure" keys (first digit > D1;
//      fewer than k in the row) and its candidates (first digit == D1; on index
//      scores a few thousand in a 128K row) in shared memory -- warp scans
//      give each flagged key its slot (no atomics, no sort);
//   3. one cluster barrier; the leader appends the other CTAs' lists to its
//      own (distributed shared memory, rank order = index order), takes the
//      second and third digits from the candidates, selects them (key > T,
//      then the lowest-indexed keys == T: ties go to the lower index) and
//      merges them with the sure keys into the ascending output.
// Rows whose candidates or sure keys overflow the leader's lists (all-equal
// rows, rows inside one exponent bucket) take the second and third digits
// from cluster-wide histograms of every CTA's slice (merged in the leader),
// then every CTA writes its own kept keys at offsets from the lower-ranked
// CTAs' counts.  Rows with at most k candidates are written directly.
#include "dsa_common.cuh"
#include "dsa_internal.h"

namespace dsa {
namespace {

constexpr int kThreads = 512;
constexpr int kPer = 16;                   // keys a thread in a chunk
constexpr int kSteps = kPer / 4;           // float4 steps a lane
constexpr int kChunk = kThreads * kPer;    // keys a chunk: 8192
constexpr int kCtaChunks = 2;              // chunks a CTA of a cluster takes
constexpr int kSlice = kCtaChunks * kChunk;  // keys a CTA of a cluster: 16384
constexpr int kWarps = kThreads / 32;
constexpr int kMaxCluster = 16;
constexpr int kBins1 = 2048;               // first and second digits: 11 bits
constexpr int kBins3 = 1024;               // third digit: 10 bits
constexpr int kListCap = 4096;             // leader's sure / candidate list capacity

// ------------------------------------------------- distributed shared memory --
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// The address of `p` (this CTA's shared memory) in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t map_rank(const void* p, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_addr(p)), "r"(rank));
  return r;
}
__device__ __forceinline__ uint32_t ld_cluster(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
  return v;
}
__device__ __forceinline__ void red_add_cluster(uint32_t addr, uint32_t v) {
  asm volatile("red.relaxed.cluster.shared::cluster.add.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}
__device__ __forceinline__ void cluster_arrive() {
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() {
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_sync() {
  cluster_arrive();
  cluster_wait();
}

// ------------------------------------------------------------------ scans --
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
// *total.  Uses `wsum` (kWarps + 1 words); ends with a barrier.
__device__ __forceinline__ uint32_t block_excl_scan(uint32_t v, uint32_t* wsum, uint32_t* total) {
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

// The bin of `hist` (nbins, counted from the top) that holds the
// `remaining`-th largest key: *digit, and *above = keys in higher bins.
__device__ __forceinline__ void select_bin(const uint32_t* hist, int nbins, uint32_t remaining, uint32_t* wsum,
                                           uint32_t* s_digit, uint32_t* s_above) {
  const int bpt = nbins / kThreads;  // bins a thread, taken from the top
  const int top = nbins - 1 - static_cast<int>(threadIdx.x) * bpt;
  uint32_t cnt = 0;
  for (int i = 0; i < bpt; ++i) cnt += hist[top - i];
  uint32_t total;
  const uint32_t excl = block_excl_scan(cnt, wsum, &total);
  if (excl < remaining && remaining <= excl + cnt) {
    uint32_t cum = excl;
    for (int i = 0; i < bpt; ++i) {
      const uint32_t h = hist[top - i];
      if (remaining <= cum + h) {
        *s_digit = static_cast<uint32_t>(top - i);
        *s_above = cum;
        break;
      }
      cum += h;
    }
  }
  __syncthreads();
}

// Slots, in index order, of this thread's keys flagged in two sets (bit q =
// key q of the thread: step q / 4, element q % 4 of the layout at key_pos).
// Packed warp scans (four 8-bit step counts a word) order a warp's keys by
// step, lane, element; one block scan orders the warps.
struct Slots {
  uint32_t sa, sb;  // exclusive scans over lanes of the step counts (a byte a step)
  uint32_t ta, tb;  // the warp's step totals (a byte a step)
  uint32_t base;    // keys of earlier warps (a << 16 | b)
  __device__ __forceinline__ static uint32_t field(uint32_t w, int i) { return (w >> (8 * i)) & 0xFFu; }
  // the bytes of steps 0..i-1 summed (i <= 4; a byte never carries: a step
  // has at most 128 keys a warp)
  __device__ __forceinline__ static uint32_t before(uint32_t t, int i) {
    const uint32_t low = i == 0 ? 0u : (t & (0xFFFFFFFFu >> (32 - 8 * i)));
    return (low & 0xFFu) + ((low >> 8) & 0xFFu) + ((low >> 16) & 0xFFu) + (low >> 24);
  }
  // slot (from the chunk's first key) of this thread's first set-a / set-b key of step i
  __device__ __forceinline__ uint32_t a(int i) const { return (base >> 16) + before(ta, i) + field(sa, i); }
  __device__ __forceinline__ uint32_t b(int i) const { return (base & 0xFFFFu) + before(tb, i) + field(sb, i); }
};

// Fills *S for the flag sets fa, fb; returns the CTA's totals (a << 16 | b).
__device__ __forceinline__ uint32_t order_slots(uint32_t fa, uint32_t fb, Slots* S, uint32_t* wsum) {
  static_assert(kSteps == 4, "one packed word of step counts");
  const int lane = lane_id(), warp = threadIdx.x >> 5;
  uint32_t ca = 0, cb = 0;
#pragma unroll
  for (int i = 0; i < kSteps; ++i) {
    ca |= static_cast<uint32_t>(__popc((fa >> (4 * i)) & 0xFu)) << (8 * i);
    cb |= static_cast<uint32_t>(__popc((fb >> (4 * i)) & 0xFu)) << (8 * i);
  }
  const uint32_t ia = warp_incl_scan(ca), ib = warp_incl_scan(cb);
  S->sa = ia - ca;
  S->sb = ib - cb;
  S->ta = __shfl_sync(0xffffffffu, ia, 31);
  S->tb = __shfl_sync(0xffffffffu, ib, 31);
  const uint32_t wa = Slots::before(S->ta, 4);  // the warp's totals
  const uint32_t wb = Slots::before(S->tb, 4);
  if (lane == 0) wsum[warp] = (wa << 16) | wb;
  __syncthreads();
  if (warp == 0) {
    const uint32_t x = lane < kWarps ? wsum[lane] : 0u;
    const uint32_t xi = warp_incl_scan(x);
    if (lane < kWarps) wsum[lane] = xi - x;
    if (lane == 31) wsum[kWarps] = xi;
  }
  __syncthreads();
  S->base = wsum[warp];
  const uint32_t total = wsum[kWarps];
  __syncthreads();
  return total;
}

struct RowSel {
  const float* scores;
  int64_t ld;
  const int32_t* ctx_len;
  const int32_t* q_pos0;
  int t_off, n_q, s_max, k, C;
  int32_t* idx;
  const int32_t* remap;        // output idx = remap[row * remap_ld + s] (or s when null)
  int64_t remap_ld;
  const uint32_t* hist_parts;  // the indexer's partial first-digit histograms, or null
  int hist_per_cta, hist_tpr;
};

// Shared memory of one CTA (the same layout in every CTA of a cluster).
struct TopkSmem {
  uint32_t hist[kBins1];     // the row's first-digit histogram; later scratch for local counts
  uint32_t hsum[kBins1];     // leader: the cluster's first-digit counts (when counted here)
  uint32_t h2sum[kBins1];    // leader: the cluster's second-digit counts (overflow rows)
  uint32_t h3sum[kBins3];    // leader: the cluster's third-digit counts
  uint32_t wsum[kWarps + 1];
  uint32_t res[8];
  uint32_t meta[4];          // this CTA's list sizes and kept-key counts, read by the others
  int32_t sure[kListCap];
  int32_t selc[kListCap];
  uint32_t ckey[kListCap];
  int32_t cidx[kListCap];
};

__global__ void __launch_bounds__(kThreads, 2) topk_cluster_kernel(RowSel P) {
  pdl_wait();
  extern __shared__ __align__(16) uint8_t smem_raw[];
  TopkSmem& sm = *reinterpret_cast<TopkSmem*>(smem_raw);
  const int C = P.C;
  const uint32_t c = cluster_rank();
  const int r = blockIdx.x / C;
  const int b = r / P.n_q, t = r % P.n_q;
  const int L = min(max(__ldg(P.ctx_len + b), 0), P.s_max);
  const int n = max(0, min(__ldg(P.q_pos0 + b) + P.t_off + t + 1, L));  // candidates s in [0, n)
  int32_t* out = P.idx + static_cast<int64_t>(r) * P.k;
  const int32_t* remap = P.remap ? P.remap + static_cast<int64_t>(r) * P.remap_ld : nullptr;
  const float* row = P.scores + static_cast<int64_t>(r) * P.ld;
  const int tid = threadIdx.x, lane = lane_id(), warp = tid >> 5;
  auto emit = [&](int pos, int s) { out[pos] = remap ? __ldg(remap + s) : s; };

  if (n <= P.k) {  // the same in every CTA of the cluster: nobody syncs
    for (int j = static_cast<int>(c) * kThreads + tid; j < P.k; j += C * kThreads) {
      if (j < n) emit(j, j);
      else out[j] = -1;
    }
    pdl_trigger();
    return;
  }

  // ---- the keys: with C > 1, CTA c takes the slice [c kSlice, (c + 1) kSlice)
  // as two chunks; with C == 1 the CTA walks the row in chunks of kChunk keys.
  // In a chunk, warp w covers [w 32 kPer, (w + 1) 32 kPer) and step i of lane
  // l holds the four keys 4 (32 i + l) + e of that range.
  const int nch = C > 1 ? kCtaChunks : (n + kChunk - 1) / kChunk;
  int cbase = C > 1 ? static_cast<int>(c) * kSlice : 0;
  auto key_pos = [&](int i, int e) { return cbase + warp * (32 * kPer) + 4 * (32 * i + lane) + e; };
  // (keys are loaded again where a later phase needs them, rather than kept
  // live across the scans: the reloads hit L1/L2)
  auto load_slice = [&](uint32_t* key) -> uint32_t {
    uint32_t m = 0;
#pragma unroll
    for (int i = 0; i < kSteps; ++i) {
      const int p0 = key_pos(i, 0);
      if (p0 + 4 <= n) {
        const float4 f = __ldg(reinterpret_cast<const float4*>(row + p0));
        key[4 * i] = float_order_key(f.x);
        key[4 * i + 1] = float_order_key(f.y);
        key[4 * i + 2] = float_order_key(f.z);
        key[4 * i + 3] = float_order_key(f.w);
        m |= 0xFu << (4 * i);
      } else {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const bool v = p0 + e < n;
          key[4 * i + e] = v ? float_order_key(__ldg(row + p0 + e)) : 0u;
          m |= (v ? 1u : 0u) << (4 * i + e);
        }
      }
    }
    return m;
  };
  auto chunk = [&](int ch) { cbase = (C > 1 ? static_cast<int>(c) * kCtaChunks + ch : ch) * kChunk; };
  uint32_t key[kPer];
  uint32_t vm = 0;
  for (int i = tid; i < kBins1; i += kThreads) {
    sm.hist[i] = 0;
    sm.hsum[i] = 0;
    sm.h2sum[i] = 0;
  }
  for (int i = tid; i < kBins3; i += kThreads) sm.h3sum[i] = 0;
  __syncthreads();
  if (C > 1) cluster_sync();  // every CTA's sums are zero before any remote add

  // ---- 1. first digit: the row's histogram in sm.hist of every CTA
  if (P.hist_parts != nullptr) {
    // row r's key tiles [r tpr, (r + 1) tpr) were scored by the indexer CTAs
    // i_lo..i_hi (runs of per_cta tiles); CTA i kept this row in slot 0 if
    // its run starts in it, else in slot 1
    const int64_t tile0 = static_cast<int64_t>(r) * P.hist_tpr;
    const int i_lo = static_cast<int>(tile0 / P.hist_per_cta);
    const int i_hi = static_cast<int>((tile0 + P.hist_tpr - 1) / P.hist_per_cta);
    constexpr int kBpt = kBins1 / kThreads;  // bins a thread
    constexpr int kParts = 8;                // partials whose loads are in flight together
    uint32_t v[kBpt];
#pragma unroll
    for (int j = 0; j < kBpt; ++j) v[j] = 0;
    for (int i0 = i_lo; i0 <= i_hi; i0 += kParts) {
      uint32_t x[kParts][kBpt];
#pragma unroll
      for (int u = 0; u < kParts; ++u) {
        const int i = i0 + u;
        const int slot = (static_cast<int64_t>(i) * P.hist_per_cta) / P.hist_tpr == r ? 0 : 1;
        const uint32_t* src = P.hist_parts + (static_cast<int64_t>(i) * 2 + slot) * kBins1 + tid;
#pragma unroll
        for (int j = 0; j < kBpt; ++j) x[u][j] = i <= i_hi ? __ldg(src + j * kThreads) : 0u;
      }
#pragma unroll
      for (int u = 0; u < kParts; ++u)
#pragma unroll
        for (int j = 0; j < kBpt; ++j) v[j] += x[u][j];
    }
#pragma unroll
    for (int j = 0; j < kBpt; ++j) sm.hist[tid + j * kThreads] = v[j];
    __syncthreads();
  } else {
    for (int ch = 0; ch < nch; ++ch) {
      chunk(ch);
      vm = load_slice(key);
#pragma unroll
      for (int q = 0; q < kPer; ++q)
        if ((vm >> q) & 1u) atomicAdd(&sm.hist[key[q] >> 21], 1u);
    }
    __syncthreads();
    if (C > 1) {
      // merge into the leader, then every CTA copies the row's histogram
      const uint32_t lead = map_rank(sm.hsum, 0);
      for (int i = tid; i < kBins1; i += kThreads)
        if (sm.hist[i]) red_add_cluster(lead + 4u * i, sm.hist[i]);
      cluster_sync();
      for (int i = tid; i < kBins1; i += kThreads) sm.hist[i] = ld_cluster(lead + 4u * i);
      __syncthreads();
    }
  }
  select_bin(sm.hist, kBins1, static_cast<uint32_t>(P.k), sm.wsum, &sm.res[0], &sm.res[1]);
  const uint32_t D1 = sm.res[0];
  const uint32_t above1 = sm.res[1];  // sure keys of the row (first digit > D1)
  const uint32_t ncand = sm.hist[D1];
  const bool fits = ncand <= static_cast<uint32_t>(kListCap) && above1 <= static_cast<uint32_t>(kListCap) &&
                    static_cast<uint32_t>(P.k) - above1 <= static_cast<uint32_t>(kListCap);

  if (fits) {
    // ---- 2. sure keys and candidates of this CTA's keys, in index order
    uint32_t own_s = 0, own_c = 0;
    for (int ch = 0; ch < nch; ++ch) {
      chunk(ch);
      vm = load_slice(key);
      uint32_t fs = 0, fc = 0;  // sure / candidate flags
#pragma unroll
      for (int q = 0; q < kPer; ++q) {
        const uint32_t d = key[q] >> 21;
        fs |= (((vm >> q) & 1u) && d > D1) ? (1u << q) : 0u;
        fc |= (((vm >> q) & 1u) && d == D1) ? (1u << q) : 0u;
      }
      Slots S;
      const uint32_t tot = order_slots(fs, fc, &S, sm.wsum);
#pragma unroll
      for (int i = 0; i < kSteps; ++i) {
        uint32_t ps = own_s + S.a(i), pc = own_c + S.b(i);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int q = 4 * i + e;
          if ((fs >> q) & 1u) {
            sm.sure[ps++] = key_pos(i, e);
          } else if ((fc >> q) & 1u) {
            const int sp = key_pos(i, e);
            sm.ckey[pc] = float_order_key(__ldg(row + sp));
            sm.cidx[pc] = sp;
            ++pc;
          }
        }
      }
      own_s += tot >> 16;
      own_c += tot & 0xFFFFu;
    }
    if (tid == 0) {
      sm.meta[0] = own_s;
      sm.meta[1] = own_c;
    }
    __syncthreads();
    if (C > 1) {
      cluster_sync();  // lists and counts published
      if (c != 0) {
        pdl_trigger();
        cluster_sync();  // the leader reads our lists; we leave once it is done
        return;
      }
      // ---- 3. (leader) append the other CTAs' lists, in rank order: every
      // CTA's list sizes in one round of remote loads, their offsets by a
      // warp scan, then all entries pulled at once (one thread an entry)
      if (tid < 32) {
        uint32_t ps_n = 0, pc_n = 0;
        if (tid < C) {
          const uint32_t mp = map_rank(sm.meta, tid);
          ps_n = ld_cluster(mp);
          pc_n = ld_cluster(mp + 4);
        }
        const uint32_t is = warp_incl_scan(ps_n), ic = warp_incl_scan(pc_n);
        if (tid < C) {
          sm.wsum[tid] = is - ps_n;                               // sure offsets of each CTA
          reinterpret_cast<uint32_t*>(sm.selc)[tid] = ic - pc_n;  // candidate offsets (selc is free until the end)
        }
      }
      __syncthreads();
      const uint32_t* s_off = sm.wsum;
      const uint32_t* c_off = reinterpret_cast<const uint32_t*>(sm.selc);
      // entries [off(p), off(p + 1)) of the merged lists come from CTA p
      for (uint32_t j = own_s + tid; j < above1; j += kThreads) {
        int p = 1;
        while (p + 1 < C && s_off[p + 1] <= j) ++p;
        sm.sure[j] = static_cast<int32_t>(ld_cluster(map_rank(sm.sure, p) + 4u * (j - s_off[p])));
      }
      for (uint32_t j = own_c + tid; j < ncand; j += kThreads) {
        int p = 1;
        while (p + 1 < C && c_off[p + 1] <= j) ++p;
        sm.ckey[j] = ld_cluster(map_rank(sm.ckey, p) + 4u * (j - c_off[p]));
        sm.cidx[j] = static_cast<int32_t>(ld_cluster(map_rank(sm.cidx, p) + 4u * (j - c_off[p])));
      }
      __syncthreads();
      cluster_arrive();  // done with the other CTAs' shared memory
    }
    // second and third digits from the candidates (all in this CTA now)
    for (int i = tid; i < kBins1; i += kThreads) sm.hist[i] = 0;
    __syncthreads();
    for (uint32_t i = tid; i < ncand; i += kThreads) atomicAdd(&sm.hist[(sm.ckey[i] >> 10) & 0x7FFu], 1u);
    __syncthreads();
    const uint32_t rem1 = static_cast<uint32_t>(P.k) - above1;
    select_bin(sm.hist, kBins1, rem1, sm.wsum, &sm.res[2], &sm.res[3]);
    const uint32_t pref22 = (D1 << 11) | sm.res[2];
    const uint32_t rem2 = rem1 - sm.res[3];
    for (uint32_t i = tid; i < ncand; i += kThreads) {
      const uint32_t kk = sm.ckey[i];
      if ((kk >> 10) == pref22) atomicAdd(&sm.h3sum[kk & 0x3FFu], 1u);
    }
    __syncthreads();
    select_bin(sm.h3sum, kBins3, rem2, sm.wsum, &sm.res[4], &sm.res[5]);
    const uint32_t T = (pref22 << 10) | sm.res[4];
    const uint32_t take_eq = rem2 - sm.res[5];  // keys == T to keep, lowest index first
    pdl_trigger();
    // selected candidates, in index order: key > T, or key == T among the
    // first take_eq of them
    constexpr int kCPT = kListCap / kThreads;  // candidates a thread, consecutive
    const int c0 = tid * kCPT;
    uint32_t gt = 0, eq = 0;
#pragma unroll
    for (int e = 0; e < kCPT; ++e) {
      const int i = c0 + e;
      if (i < static_cast<int>(ncand)) {
        gt += sm.ckey[i] > T ? 1u : 0u;
        eq += sm.ckey[i] == T ? 1u : 0u;
      }
    }
    uint32_t tt;
    const uint32_t pre = block_excl_scan((gt << 16) | eq, sm.wsum, &tt);
    uint32_t eq_rank = pre & 0xFFFFu;
    uint32_t pos = (pre >> 16) + min(eq_rank, take_eq);
#pragma unroll
    for (int e = 0; e < kCPT; ++e) {
      const int i = c0 + e;
      if (i >= static_cast<int>(ncand)) break;
      const uint32_t kk = sm.ckey[i];
      if (kk > T) {
        sm.selc[pos++] = sm.cidx[i];
      } else if (kk == T) {
        if (eq_rank < take_eq) sm.selc[pos++] = sm.cidx[i];
        ++eq_rank;
      }
    }
    __syncthreads();
    // merge the two ascending lists: each entry's output slot is its own rank
    // plus the number of entries of the other list below it
    const int n_sure = static_cast<int>(above1);
    const int n_sel = P.k - n_sure;
    for (int i = tid; i < n_sure + n_sel; i += kThreads) {
      const bool from_sure = i < n_sure;
      const int j = from_sure ? i : i - n_sure;
      const int sv = from_sure ? sm.sure[j] : sm.selc[j];
      const int32_t* other = from_sure ? sm.selc : sm.sure;
      int lo = 0, hi = from_sure ? n_sel : n_sure;  // count of `other` entries < sv
      while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (other[mid] < sv) lo = mid + 1;
        else hi = mid;
      }
      emit(j + lo, sv);
    }
    if (C > 1) cluster_wait();
    return;
  }

  // ---- overflow: the remaining digits from histograms of every CTA's keys,
  // merged in the leader (h2sum, h3sum; with C == 1 the CTA's own)
  const uint32_t lead2 = map_rank(sm.h2sum, 0), lead3 = map_rank(sm.h3sum, 0);
  // every thread has taken ncand from sm.hist before it is cleared: a warp
  // that read a cleared bin would take the fits branch on its own
  __syncthreads();
  for (int i = tid; i < kBins1; i += kThreads) sm.hist[i] = 0;
  __syncthreads();
  for (int ch = 0; ch < nch; ++ch) {
    chunk(ch);
    vm = load_slice(key);
#pragma unroll
    for (int q = 0; q < kPer; ++q)
      if (((vm >> q) & 1u) && (key[q] >> 21) == D1) atomicAdd(&sm.hist[(key[q] >> 10) & 0x7FFu], 1u);
  }
  __syncthreads();
  for (int i = tid; i < kBins1; i += kThreads)
    if (sm.hist[i]) red_add_cluster(lead2 + 4u * i, sm.hist[i]);
  if (C > 1) cluster_sync();
  else __syncthreads();
  for (int i = tid; i < kBins1; i += kThreads) sm.hist[i] = ld_cluster(lead2 + 4u * i);
  __syncthreads();
  const uint32_t rem1 = static_cast<uint32_t>(P.k) - above1;
  select_bin(sm.hist, kBins1, rem1, sm.wsum, &sm.res[2], &sm.res[3]);
  const uint32_t pref22 = (D1 << 11) | sm.res[2];
  const uint32_t rem2 = rem1 - sm.res[3];
  for (int i = tid; i < kBins1; i += kThreads) sm.hist[i] = 0;
  __syncthreads();
  for (int ch = 0; ch < nch; ++ch) {
    chunk(ch);
    vm = load_slice(key);
#pragma unroll
    for (int q = 0; q < kPer; ++q)
      if (((vm >> q) & 1u) && (key[q] >> 10) == pref22) atomicAdd(&sm.hist[key[q] & 0x3FFu], 1u);
  }
  __syncthreads();
  for (int i = tid; i < kBins3; i += kThreads)
    if (sm.hist[i]) red_add_cluster(lead3 + 4u * i, sm.hist[i]);
  if (C > 1) cluster_sync();
  else __syncthreads();
  for (int i = tid; i < kBins3; i += kThreads) sm.hist[i] = ld_cluster(lead3 + 4u * i);
  __syncthreads();
  select_bin(sm.hist, kBins3, rem2, sm.wsum, &sm.res[4], &sm.res[5]);
  const uint32_t T = (pref22 << 10) | sm.res[4];
  const uint32_t take_eq = rem2 - sm.res[5];
  pdl_trigger();
  // every CTA writes its kept keys: keys > T, and keys == T while fewer than
  // take_eq have been kept; offsets from the lower-ranked CTAs' counts (C > 1)
  // or from the earlier chunks (C == 1)
  uint32_t gt_off = 0, eq_off = 0;
  if (C > 1) {
    uint32_t ng = 0, ne = 0;
    for (int ch = 0; ch < nch; ++ch) {
      chunk(ch);
      vm = load_slice(key);
#pragma unroll
      for (int q = 0; q < kPer; ++q) {
        ng += (((vm >> q) & 1u) && key[q] > T) ? 1u : 0u;
        ne += (((vm >> q) & 1u) && key[q] == T) ? 1u : 0u;
      }
    }
    uint32_t tt;
    block_excl_scan((ng << 16) | ne, sm.wsum, &tt);
    if (tid == 0) {
      sm.meta[2] = tt >> 16;
      sm.meta[3] = tt & 0xFFFFu;
    }
    __syncthreads();
    cluster_sync();
    if (tid < 32) {
      uint32_t g = 0, e = 0;
      if (tid < static_cast<int>(c)) {
        const uint32_t mp = map_rank(sm.meta, tid);
        g = ld_cluster(mp + 8);
        e = ld_cluster(mp + 12);
      }
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        g += __shfl_xor_sync(0xffffffffu, g, off);
        e += __shfl_xor_sync(0xffffffffu, e, off);
      }
      if (tid == 0) {
        sm.res[6] = g;
        sm.res[7] = e;
      }
    }
    __syncthreads();
    gt_off = sm.res[6];
    eq_off = sm.res[7];
    cluster_arrive();  // done reading the other CTAs' counts
  }
  for (int ch = 0; ch < nch; ++ch) {
    chunk(ch);
    vm = load_slice(key);
    uint32_t fg = 0, fe = 0;
#pragma unroll
    for (int q = 0; q < kPer; ++q) {
      fg |= (((vm >> q) & 1u) && key[q] > T) ? (1u << q) : 0u;
      fe |= (((vm >> q) & 1u) && key[q] == T) ? (1u << q) : 0u;
    }
    Slots S;
    const uint32_t tot = order_slots(fg, fe, &S, sm.wsum);
#pragma unroll
    for (int i = 0; i < kSteps; ++i) {
      uint32_t gtc = gt_off + S.a(i), eqc = eq_off + S.b(i);  // keys > T / == T of the row before this one
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int q = 4 * i + e;
        if ((fg >> q) & 1u) {
          emit(gtc + min(eqc, take_eq), key_pos(i, e));
          ++gtc;
        } else if ((fe >> q) & 1u) {
          if (eqc < take_eq) emit(gtc + eqc, key_pos(i, e));
          ++eqc;
        }
      }
    }
    gt_off += tot >> 16;
    eq_off += tot & 0xFFFFu;
  }
  if (C > 1) cluster_wait();  // nobody leaves while another CTA may read its counts
}

}  // namespace

size_t topk_workspace_bytes(int, int, int, int) { return 0; }

dsa_status_t topk_radix(const TopkArgs& a) {
  const int64_t rows = static_cast<int64_t>(a.B) * a.n_q;
  if (rows == 0) return DSA_OK;
  static_assert(kSlice < 65536, "per-CTA counts are packed in 16 bits");
  static_assert(kListCap % kThreads == 0, "candidates a thread");
  const int64_t n_max = std::max(1, a.s_max);
  int64_t C = (n_max + kSlice - 1) / kSlice;
  // many rows (prefill rounds): a CTA a row, walking it in chunks, so that
  // many rows are in flight; few long rows (decode): a cluster a row
  if (rows >= 2LL * std::max(1, device_sm_count(a.device))) C = 1;
  if (C > kMaxCluster) return DSA_ERR_UNSUPPORTED;
  if (rows * C > INT32_MAX) return DSA_ERR_UNSUPPORTED;
  if ((reinterpret_cast<uintptr_t>(a.scores) & 15u) != 0 || (a.ld & 3) != 0) return DSA_ERR_INVALID_ARG;
  RowSel P;
  P.scores = a.scores;
  P.ld = a.ld;
  P.ctx_len = a.ctx_len;
  P.q_pos0 = a.q_pos0;
  P.t_off = a.t_off;
  P.n_q = a.n_q;
  P.s_max = a.s_max;
  P.k = a.k;
  P.C = static_cast<int>(C);
  P.idx = a.idx;
  P.remap = a.remap;
  P.remap_ld = a.remap_ld;
  P.hist_parts = a.hist_parts;
  P.hist_per_cta = a.hist_per_cta;
  P.hist_tpr = a.hist_tpr;
  if (P.hist_parts != nullptr && (P.hist_per_cta <= 0 || P.hist_tpr <= 0)) return DSA_ERR_INVALID_ARG;
  const size_t smem = sizeof(TopkSmem);
  static bool attr_done[64] = {};
  if (a.device < 0 || a.device >= 64) return DSA_ERR_UNSUPPORTED;
  if (!attr_done[a.device]) {
    if (cudaFuncSetAttribute(topk_cluster_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem)) != cudaSuccess ||
        cudaFuncSetAttribute(topk_cluster_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) !=
            cudaSuccess)
      return DSA_ERR_CUDA;
    attr_done[a.device] = true;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(rows * C), 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = a.stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = static_cast<unsigned>(C);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1] = pdl_attribute();
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, topk_cluster_kernel, P) == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

}  // namespace dsa
