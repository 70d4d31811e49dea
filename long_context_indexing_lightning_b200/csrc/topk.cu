// Fine-grained token selection: per query, the index_topk best-scored
// previous keys (DeepSeek-V3.2 model doc, Transformers, section "DeepSeek
// Sparse Attention (DSA)", item 2; index_topk defaults to 2048).
//
// Radix select on order-preserving 32-bit keys, no sort.  One query row is
// split over a thread-block cluster of C CTAs (C = 1..16, 16K keys a CTA in
// two chunks of 8K, read with coalesced loads); when a launch has many rows
// (prefill), C = 1 and each CTA walks its row chunk by chunk.  The key splits
// into digits of 11, 11 and 10 bits; T, the key of the k-th largest score, is
// found digit by digit:
//   1. the first digit's histogram: summed from the partial histograms the
//      indexer's epilogue built (TopkArgs::hist_parts) straight into
//      registers, or counted by each CTA and merged in the cluster's first
//      CTA (the leader); every CTA finds the bin D1 holding the k-th largest
//      key, the keys above it and the keys in it;
//   2. each CTA lists its keys with first digit >= D1 (the sure keys above D1
//      and the candidates in it) in index order in its shared memory: a
//      chunk's keys are ordered by warp scans (no sort, no atomics), and the
//      candidates' second digits are counted on the way;
//   3. the second and third digits: each CTA adds its counts into the
//      leader's histograms (remote atomics, one cluster barrier each) and
//      every CTA selects the digit from them; only the few listed keys in the
//      second digit's bin are read again for their third digit;
//   4. each CTA counts its kept keys (key > T, then the lowest-indexed keys ==
//      T: ties go to the lower index), learns the lower-ranked CTAs' counts
//      through the leader, and writes its kept keys into its own range of the
//      ascending output, warps ranking the list with ballots.
// A list entry is one word: bit 31 = sure key (first digit > D1), bits 19..29
// = the second digit (after the third-digit pass, for the entries in the
// second digit's bin D2: the third digit, flagged by bit 30), bits 13..18 =
// the chunk of the CTA's walk, bits 0..12 = the key's offset in that chunk.
// A CTA of a cluster lists at most its own 16K keys, so every clustered row
// fits.  A single CTA whose row lists more keys than its list holds
// (all-equal rows, rows inside one exponent bucket) takes the second and
// third digits from histograms of the whole row and writes its kept keys
// chunk by chunk.  Rows with at most k candidates are written directly.
//
// The handed-over partial histograms are checked against the scores: a
// mismatch (a histogram from another call) records DSA_ERR_HIST_MISMATCH in
// the device error word and leaves the row's output undefined, never an
// access out of bounds.
#include "dsa_common.cuh"
#include "dsa_internal.h"

namespace dsa {
namespace {

constexpr int kThreads = 512;
constexpr int kPer = 16;                   // keys a thread in a chunk
constexpr int kSteps = kPer / 4;           // float4 steps a lane
constexpr int kChunk = kThreads * kPer;    // keys a chunk: 8192
// Two instances: clustered rows (decode) with CTAs of 4 chunks (32K keys, one
// CTA an SM, the slice brought into shared memory by one bulk copy), and one
// CTA walking a row (many rows: two CTAs an SM, keys read chunk by chunk).
constexpr int kClusterChunks = 4;          // chunks a CTA of a cluster takes
constexpr int kClusterSlice = kClusterChunks * kChunk;  // keys a CTA of a cluster: 32768
constexpr int kWarps = kThreads / 32;
constexpr int kMaxCluster = 16;
constexpr int kBins1 = 2048;               // first and second digits: 11 bits
constexpr int kBins3 = 1024;               // third digit: 10 bits
constexpr int kListCapCluster = kClusterSlice;  // a clustered CTA lists at most its slice
constexpr int kListCapRow = 16384;         // a CTA walking a row: longer lists take the overflow path
constexpr uint32_t kNoBin = 0xFFFFFFFFu;   // select found no bin: the counts do not add up
constexpr uint32_t kSure = 1u << 31;       // list entry: first digit > D1
constexpr uint32_t kHasD3 = 1u << 30;      // list entry: bits 19..29 hold the third digit
constexpr uint32_t kOffMask = kChunk - 1;  // list entry: offset in the chunk
constexpr uint32_t kPosMask = (0x3Fu << 13) | kOffMask;  // list entry: chunk and offset
constexpr int kBndCap = 64;                // boundary keys (second digit == D2) a row resolves directly
static_assert(kChunk == 8192, "13-bit chunk offsets");

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
__device__ __forceinline__ uint4 ld_cluster_v4(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared::cluster.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr)
               : "memory");
  return v;
}
__device__ __forceinline__ uint32_t ld_cluster(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
  return v;
}
__device__ __forceinline__ void st_cluster(uint32_t addr, uint32_t v) {
  asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}
__device__ __forceinline__ void red_add_cluster(uint32_t addr, uint32_t v) {
  asm volatile("red.relaxed.cluster.shared::cluster.add.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}
__device__ __forceinline__ void cluster_arrive() {
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
// Arrival that publishes nothing (this CTA's earlier writes are its own).
__device__ __forceinline__ void cluster_arrive_relaxed() {
  asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() {
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_sync() {
  cluster_arrive();
  cluster_wait();
}
__device__ __forceinline__ uint32_t lanemask_lt() {
  uint32_t m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
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

// The bin holding the `remaining`-th largest key of a histogram of
// kBpt * kThreads bins, thread t holding the counts of bins top - j (j <
// kBpt, top = bins - 1 - t kBpt) in h[j].  Writes res[0] = the bin (kNoBin if
// the counts add up to fewer than `remaining`), res[1] = keys in higher bins,
// res[2] = keys in the bin.  Ends with a barrier.
template <int kBpt>
__device__ __forceinline__ void select_bin(const uint32_t (&h)[kBpt], uint32_t remaining, uint32_t* wsum,
                                           uint32_t* res) {
  if (threadIdx.x == 0) {
    res[0] = kNoBin;
    res[1] = 0;
    res[2] = 0;
  }
  uint32_t cnt = 0;
#pragma unroll
  for (int j = 0; j < kBpt; ++j) cnt += h[j];
  uint32_t total;
  const uint32_t excl = block_excl_scan(cnt, wsum, &total);  // (its barriers order the defaults first)
  if (excl < remaining && remaining <= excl + cnt) {
    uint32_t cum = excl;
    bool done = false;
#pragma unroll
    for (int j = 0; j < kBpt; ++j) {
      if (!done && remaining <= cum + h[j]) {
        res[0] = static_cast<uint32_t>(kBpt * kThreads - 1 - static_cast<int>(threadIdx.x) * kBpt - j);
        res[1] = cum;
        res[2] = h[j];
        done = true;
      }
      cum += h[j];
    }
  }
  __syncthreads();
}

// This thread's counts of a shared histogram in select_bin's order.
__device__ __forceinline__ void my_bins4(const uint32_t* hist, uint32_t (&h)[4]) {
  const uint4 v = *reinterpret_cast<const uint4*>(hist + kBins1 - 4 - 4 * threadIdx.x);
  h[0] = v.w;
  h[1] = v.z;
  h[2] = v.y;
  h[3] = v.x;
}
__device__ __forceinline__ void my_bins2(const uint32_t* hist, uint32_t (&h)[2]) {
  const uint2 v = *reinterpret_cast<const uint2*>(hist + kBins3 - 2 - 2 * threadIdx.x);
  h[0] = v.y;
  h[1] = v.x;
}

// Packed step counts (a byte a step of kSteps keys-of-4): bit q of `f` is key
// q of the thread (step q / 4, element q % 4 of the layout at key_pos).
__device__ __forceinline__ uint32_t step_counts(uint32_t f) {
  uint32_t c = 0;
#pragma unroll
  for (int i = 0; i < kSteps; ++i) c |= static_cast<uint32_t>(__popc((f >> (4 * i)) & 0xFu)) << (8 * i);
  return c;
}
// The bytes of steps 0..i-1 of a packed word summed (i <= 4; a byte never
// carries: a step has at most 128 keys a warp).
__device__ __forceinline__ uint32_t bytes_before(uint32_t t, int i) {
  const uint32_t low = i == 0 ? 0u : (t & (0xFFFFFFFFu >> (32 - 8 * i)));
  return (low & 0xFFu) + ((low >> 8) & 0xFFu) + ((low >> 16) & 0xFFu) + (low >> 24);
}
__device__ __forceinline__ uint32_t byte_of(uint32_t w, int i) { return (w >> (8 * i)) & 0xFFu; }

// Slots, in index order, of this thread's keys flagged in two sets (overflow
// rows): packed warp scans order a warp's keys by step, lane, element; one
// block scan orders the warps.
struct Slots {
  uint32_t sa, sb;  // exclusive scans over lanes of the step counts (a byte a step)
  uint32_t ta, tb;  // the warp's step totals (a byte a step)
  uint32_t base;    // keys of earlier warps (a << 16 | b)
  // slot (from the chunk's first key) of this thread's first set-a / set-b key of step i
  __device__ __forceinline__ uint32_t a(int i) const { return (base >> 16) + bytes_before(ta, i) + byte_of(sa, i); }
  __device__ __forceinline__ uint32_t b(int i) const { return (base & 0xFFFFu) + bytes_before(tb, i) + byte_of(sb, i); }
};

// Fills *S for the flag sets fa, fb; returns the CTA's totals (a << 16 | b).
__device__ __forceinline__ uint32_t order_slots(uint32_t fa, uint32_t fb, Slots* S, uint32_t* wsum) {
  static_assert(kSteps == 4, "one packed word of step counts");
  const int lane = lane_id(), warp = threadIdx.x >> 5;
  const uint32_t ca = step_counts(fa), cb = step_counts(fb);
  const uint32_t ia = warp_incl_scan(ca), ib = warp_incl_scan(cb);
  S->sa = ia - ca;
  S->sb = ib - cb;
  S->ta = __shfl_sync(0xffffffffu, ia, 31);
  S->tb = __shfl_sync(0xffffffffu, ib, 31);
  const uint32_t wa = bytes_before(S->ta, 4);  // the warp's totals
  const uint32_t wb = bytes_before(S->tb, 4);
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
  uint32_t* err;
};

// Shared memory of one CTA (the same layout in every CTA of a cluster).
template <int kEntWords, int kBndCtas>
struct TopkSmem {
  uint32_t ent[kEntWords];   // this CTA's keys with first digit >= D1, in index order (one word each)
  uint32_t hist[kBins1];     // first-digit counts when counted here; overflow rows: second/third-digit counts
  uint32_t hsum[kBins1];     // leader: the cluster's first-digit counts (counted here, C > 1)
  uint32_t h2[kBins1];       // leader: the row's second-digit counts
  uint32_t h3[kBins3];       // leader: the row's third-digit counts
  uint32_t lh2[kBins1];      // this CTA's second-digit counts (C > 1)
  uint32_t lh3[kBins3];      // this CTA's third-digit counts (C > 1)
  uint32_t wsum[kWarps + 2];
  uint32_t res[12];          // selected digits: [0..2] first, [3..5] second, [6..8] third
  uint32_t kept[kMaxCluster];  // leader: each CTA's kept keys (keys > T << 16 | keys == T)
  uint32_t wcnt[kWarps];     // a warp's keys > T and == T (gt << 16 | eq)
  uint2 bnd[kBndCtas * kBndCap];  // leader: each CTA's boundary keys (key, index), kBndCap a CTA
  uint2 bk[kBndCap];         // the row's boundary keys, gathered from the leader
  uint32_t bslot[kBndCap];   // list slots of this CTA's boundary keys
  uint32_t kbc[kMaxCluster];  // kept boundary keys of each CTA
  uint32_t bpre[kMaxCluster];  // first slot of each CTA's boundary keys in bk
  uint32_t bcount, gdsum, found;
  uint64_t kbar;             // clustered CTAs: the slice's bulk copy landed
  int abort_flag;
};

// kCtaChunks: chunks a CTA of a cluster takes; kListCap: list entries;
// kMinBlocks: CTAs an SM.  kStaged (the clustered instance): the CTA's slice
// of the score row is copied into its list array one chunk above the front
// (one bulk copy, all of it in flight at once) and the chunks are read from
// there; after chunk ch the list holds at most (ch + 1) kChunk entries, so it
// never reaches keys not yet listed (chunk ch's keys start at (ch + 1) kChunk).
template <int kCtaChunks, int kListCap, int kMinBlocks>
__global__ void __launch_bounds__(kThreads, kMinBlocks) topk_cluster_kernel(RowSel P) {
  constexpr bool kStaged = kMinBlocks == 1;
  constexpr int kEntWords = kStaged ? kCtaChunks * kChunk + kChunk : kListCap;
  constexpr int kBndCtas = kStaged ? kMaxCluster : 1;  // (the walking instance runs one-CTA clusters)
  static_assert(!kStaged || kCtaChunks * kChunk <= kListCap, "a clustered CTA lists at most its slice");
  pdl_wait();
  extern __shared__ __align__(16) uint8_t smem_raw[];
  TopkSmem<kEntWords, kBndCtas>& sm = *reinterpret_cast<TopkSmem<kEntWords, kBndCtas>*>(smem_raw);
  const int C = P.C;
  const uint32_t c = cluster_rank();
  const bool lead = (c == 0);
  const int r = blockIdx.x / C;
  const int b = r / P.n_q, t = r % P.n_q;
  const int k = P.k;
  const int tid = threadIdx.x, lane = lane_id(), warp = tid >> 5;
  const float* row = P.scores + static_cast<int64_t>(r) * P.ld;
  const int ctx = __ldg(P.ctx_len + b), pos0 = __ldg(P.q_pos0 + b);

  // ---- issued before the row length is known: the first digit's partial
  // histograms
  uint32_t h1[4] = {0u, 0u, 0u, 0u};
  if (P.hist_parts != nullptr) {
    // row r's key tiles [r tpr, (r + 1) tpr) were scored by the indexer CTAs
    // i_lo..i_hi (runs of per_cta tiles); CTA i kept this row in slot 0 if
    // its run starts in it, else in slot 1.  This thread sums its four bins.
    const int64_t tile0 = static_cast<int64_t>(r) * P.hist_tpr;
    const int i_lo = static_cast<int>(tile0 / P.hist_per_cta);
    const int i_hi = static_cast<int>((tile0 + P.hist_tpr - 1) / P.hist_per_cta);
    constexpr int kParts = 8;  // partials whose loads are in flight together
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    for (int i0 = i_lo; i0 <= i_hi; i0 += kParts) {
      uint4 x[kParts];
#pragma unroll
      for (int u = 0; u < kParts; ++u) {
        const int i = i0 + u;
        // CTA i's run starts in this row: slot 0 (a comparison, no division)
        const int64_t run0 = static_cast<int64_t>(i) * P.hist_per_cta;
        const int slot = (run0 >= tile0 && run0 < tile0 + P.hist_tpr) ? 0 : 1;
        const uint4* src = reinterpret_cast<const uint4*>(P.hist_parts + (static_cast<int64_t>(i) * 2 + slot) * kBins1 +
                                                          (kBins1 - 4 - 4 * tid));
        x[u] = i <= i_hi ? __ldg(src) : make_uint4(0u, 0u, 0u, 0u);
      }
#pragma unroll
      for (int u = 0; u < kParts; ++u) {
        v.x += x[u].x;
        v.y += x[u].y;
        v.z += x[u].z;
        v.w += x[u].w;
      }
    }
    h1[0] = v.w;
    h1[1] = v.z;
    h1[2] = v.y;
    h1[3] = v.x;
  }

  const int L = min(max(ctx, 0), P.s_max);
  const int n = max(0, min(pos0 + P.t_off + t + 1, L));  // candidates s in [0, n)
  int32_t* out = P.idx + static_cast<int64_t>(r) * k;
  const int32_t* remap = P.remap ? P.remap + static_cast<int64_t>(r) * P.remap_ld : nullptr;
  // (a position at or past k only comes from a histogram that does not
  // describe these scores)
  auto emit = [&](uint32_t pos, int s) {
    if (pos < static_cast<uint32_t>(k)) out[pos] = remap ? __ldg(remap + s) : s;
    else raise_error(P.err, kErrHistMismatch);
  };

  if (n <= k) {  // the same in every CTA of the cluster: nobody syncs
    for (int j = static_cast<int>(c) * kThreads + tid; j < k; j += C * kThreads) {
      if (j < n) emit(j, j);
      else out[j] = -1;
    }
    pdl_trigger();
    return;
  }

  // ---- the keys: with C > 1, CTA c takes kCtaChunks chunks from chunk
  // c kCtaChunks; with C == 1 the CTA walks the row in chunks of kChunk keys.
  // In a chunk, warp w covers [w 32 kPer, (w + 1) 32 kPer) and step i of lane
  // l holds the four keys 4 (32 i + l) + e of that range.
  const int nch = C > 1 ? kCtaChunks : (n + kChunk - 1) / kChunk;
  const int chunk0 = C > 1 ? static_cast<int>(c) * kCtaChunks : 0;  // the CTA's first chunk of the row
  int cbase = chunk0 * kChunk;
  auto key_pos = [&](int i, int e) { return cbase + warp * (32 * kPer) + 4 * (32 * i + lane) + e; };
  // the keys of the chunk at `base` (this thread's kPer of them) and their
  // validity; staged: from the slice in shared memory
  const float* staged = reinterpret_cast<const float*>(sm.ent + kChunk) - chunk0 * kChunk;  // (by row position)
  auto load_at = [&](int base, uint32_t* key) -> uint32_t {
    uint32_t m = 0;
#pragma unroll
    for (int i = 0; i < kSteps; ++i) {
      const int p0 = base + warp * (32 * kPer) + 4 * (32 * i + lane);
      if (p0 + 4 <= n) {
        const float4 f = kStaged ? *reinterpret_cast<const float4*>(staged + p0)
                                 : __ldg(reinterpret_cast<const float4*>(row + p0));
        key[4 * i] = float_order_key(f.x);
        key[4 * i + 1] = float_order_key(f.y);
        key[4 * i + 2] = float_order_key(f.z);
        key[4 * i + 3] = float_order_key(f.w);
        m |= 0xFu << (4 * i);
      } else {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const bool v = p0 + e < n;
          key[4 * i + e] = v ? float_order_key(kStaged ? staged[p0 + e] : __ldg(row + p0 + e)) : 0u;
          m |= (v ? 1u : 0u) << (4 * i + e);
        }
      }
    }
    return m;
  };
  auto load_slice = [&](uint32_t* key) -> uint32_t { return load_at(cbase, key); };
  // (walking) pull chunk ch's lines into L2 ahead of its register loads, so
  // that each chunk costs an L2 round trip instead of an HBM one
  auto prefetch_chunk = [&](int ch) {
    if (!kStaged && ch < nch && tid < kChunk / 32) {
      const int p = (chunk0 + ch) * kChunk + tid * 32;
      if (p < n) asm volatile("prefetch.global.L2 [%0];" ::"l"(row + p));
    }
  };
  if constexpr (kStaged) {
    // the slice [chunk0 kChunk, + kCtaChunks kChunk) clipped to the row (to a
    // multiple of 4 keys: the row's storage is), in one bulk copy
    if (tid == 0) {
      sm.abort_flag = 0;
      const uint32_t bar = smem_addr(&sm.kbar);
      mbar_init(bar, 1);
      fence_mbar_init();
      const int lo = chunk0 * kChunk, hi = min(lo + kCtaChunks * kChunk, (n + 3) & ~3);
      if (hi > lo) {
        const uint32_t bytes = static_cast<uint32_t>(hi - lo) * 4u;
        mbar_arrive_expect_tx(bar, bytes);
        asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                         smem_addr(sm.ent + kChunk)),
                     "l"(row + lo), "r"(bytes), "r"(bar)
                     : "memory");
      } else {
        mbar_arrive(bar);
      }
    }
  }
  // (staged) every thread waits for the slice before its first key read
  bool have_slice = !kStaged;
  bool lead_arrived = false;  // (clusters) the leader's arrival at the barrier after the zeroing
  auto lead_arrive = [&]() {
    if (C > 1 && lead && !lead_arrived) {
      cluster_arrive();
      lead_arrived = true;
    }
  };
  // (every call comes after the sums below are zeroed) the leader publishes
  // its zeroed sums once its own slice has landed: a release-ordered arrival
  // with the bulk copy still in flight waited ~1 us for it
  auto wait_slice = [&]() {
    if (kStaged && !have_slice) {
      mbar_wait(smem_addr(&sm.kbar), 0, &sm.abort_flag, P.err);
      have_slice = true;
    }
    lead_arrive();
  };
  auto chunk = [&](int ch) { cbase = (chunk0 + ch) * kChunk; };
  uint32_t key[kPer];
  uint32_t vm = 0;

  // Sums start at zero: the leader's (touched by the others only after the
  // cluster barrier it arrives at once they are) and this CTA's own.
  if (lead) {
    for (int i = tid; i < kBins1; i += kThreads) {
      sm.hsum[i] = 0;
      sm.h2[i] = 0;
    }
    for (int i = tid; i < kBins3; i += kThreads) sm.h3[i] = 0;
  }
  for (int i = tid; i < kBins1; i += kThreads) {
    sm.lh2[i] = 0;
    if (P.hist_parts == nullptr) sm.hist[i] = 0;
  }
  for (int i = tid; i < kBins3; i += kThreads) sm.lh3[i] = 0;
  if (tid < kMaxCluster) sm.kbc[tid] = 0;
  if (tid == 0) {
    sm.bcount = 0;
    sm.gdsum = 0;
    sm.found = 0;
  }
  __syncthreads();
  // (only the leader's sums are read across the cluster: the others' arrivals
  // publish nothing; the leader arrives in wait_slice)
  if (C > 1 && !lead) cluster_arrive_relaxed();
  bool waited = (C == 1);
  auto wait_zeroed = [&]() {  // before the first access to the leader's sums
    if (!waited) {
      lead_arrive();
      cluster_wait();
      waited = true;
    }
  };
  // leave once nobody can still read the leader's shared memory: every CTA
  // arrives, the leader waits (every CTA of a cluster calls this at the same
  // point)
  auto leave = [&]() {
    pdl_trigger();
    if (C > 1) {
      cluster_arrive();
      if (lead) cluster_wait();
    }
  };
  // the counts do not add up (only with a mismatched histogram): flag, clear
  // the row, leave
  auto give_up = [&]() {
    if (tid == 0) raise_error(P.err, kErrHistMismatch);
    if (lead)
      for (int j = tid; j < k; j += kThreads) out[j] = -1;
  };

  // ---- 1. first digit
  if (P.hist_parts == nullptr) {
    wait_slice();
    prefetch_chunk(1);
    for (int ch = 0; ch < nch; ++ch) {
      prefetch_chunk(ch + 2);
      chunk(ch);
      vm = load_slice(key);
#pragma unroll
      for (int q = 0; q < kPer; ++q)
        if ((vm >> q) & 1u) atomicAdd(&sm.hist[key[q] >> 21], 1u);
    }
    __syncthreads();
    if (C > 1) {
      // merge into the leader; every CTA reads the row's counts back
      wait_zeroed();
      const uint32_t lsum = map_rank(sm.hsum, 0);
      for (int i = tid; i < kBins1; i += kThreads)
        if (sm.hist[i]) red_add_cluster(lsum + 4u * i, sm.hist[i]);
      cluster_sync();
      const uint4 v = ld_cluster_v4(lsum + 4u * (kBins1 - 4 - 4 * tid));
      h1[0] = v.w;
      h1[1] = v.z;
      h1[2] = v.y;
      h1[3] = v.x;
    } else {
      my_bins4(sm.hist, h1);
    }
  }
  select_bin<4>(h1, static_cast<uint32_t>(k), sm.wsum, &sm.res[0]);
  const uint32_t D1 = sm.res[0];
  const uint32_t above1 = sm.res[1];  // sure keys of the row (first digit > D1)
  const uint32_t ncand = sm.res[2];   // keys in bin D1
  if (D1 == kNoBin) {  // (every CTA read the same counts; none has touched the leader yet)
    give_up();
    wait_slice();  // (no CTA leaves with its bulk copy still landing)
    pdl_trigger();
    return;
  }
  // a CTA of a cluster lists at most its 16K keys; one CTA walking a whole
  // row must fit the row's listed keys
  const bool fits = C > 1 || above1 + ncand <= static_cast<uint32_t>(kListCap);

  if (fits) {
    // ---- 2. this CTA's keys with first digit >= D1, in index order, into
    // its list; the candidates' second digits counted on the way
    uint32_t* my_h2 = C > 1 ? sm.lh2 : sm.h2;
    uint32_t own = 0;
    // (staged) the test "first digit >= D1" on a float's raw bits b: the order
    // key is b | 2^31 for b >= 0 and ~b for b < 0 (-0 mapped like +0), so it
    // holds iff b >= pos_min (non-negative b) or b <= neg_max (negative b)
    const uint32_t K0 = D1 << 21;
    const uint32_t pos_min = K0 >= 0x80000000u ? K0 - 0x80000000u : 0u;
    const uint32_t neg_max = K0 == 0x80000000u ? 0x80000000u : ~K0;  // (K0 > 2^31: ~K0 < 2^31, no negative b)
    wait_slice();
    prefetch_chunk(1);
    for (int ch = 0; ch < nch; ++ch) {
      prefetch_chunk(ch + 2);
      chunk(ch);
      uint32_t f = 0;
      if constexpr (kStaged) {
#pragma unroll
        for (int i = 0; i < kSteps; ++i) {
          const int p0 = key_pos(i, 0);
          const uint4 u = *reinterpret_cast<const uint4*>(staged + p0);  // (past n: masked below)
          const uint32_t b[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const bool hit = static_cast<int32_t>(b[e]) >= 0 ? b[e] >= pos_min : b[e] <= neg_max;
            f |= (hit && p0 + e < n) ? (1u << (4 * i + e)) : 0u;
          }
        }
      } else {
        vm = load_slice(key);
#pragma unroll
        for (int q = 0; q < kPer; ++q) f |= (((vm >> q) & 1u) && (key[q] >> 21) >= D1) ? (1u << q) : 0u;
      }
      const uint32_t cnt = step_counts(f);
      const uint32_t inc = warp_incl_scan(cnt);
      const uint32_t sl = inc - cnt;                                  // earlier lanes, a byte a step
      const uint32_t tw = __shfl_sync(0xffffffffu, inc, 31);          // the warp's step totals
      if (lane == 0) sm.wsum[warp] = bytes_before(tw, kSteps);
      __syncthreads();
      if (warp == 0) {
        const uint32_t x = lane < kWarps ? sm.wsum[lane] : 0u;
        const uint32_t xi = warp_incl_scan(x);
        if (lane < kWarps) sm.wsum[lane] = xi - x;
        if (lane == 31) sm.wsum[kWarps] = xi;  // the chunk's listed keys
      }
      __syncthreads();
      const uint32_t wbase = own + sm.wsum[warp];
      own += sm.wsum[kWarps];
      auto put = [&](uint32_t p, uint32_t kk, int pos) {
        const bool sure = (kk >> 21) > D1;
        const uint32_t d2 = (kk >> 10) & 0x7FFu;
        if (!sure) atomicAdd(&my_h2[d2], 1u);
        if (p < static_cast<uint32_t>(kListCap))
          sm.ent[p] = (sure ? kSure : d2 << 19) | (static_cast<uint32_t>(ch) << 13) | static_cast<uint32_t>(pos - cbase);
      };
      if constexpr (kStaged) {
        // only the listed keys (a few per warp), read again from the slice
        for (uint32_t ff = f; ff != 0u; ff &= ff - 1u) {
          const int q = __ffs(ff) - 1, i = q >> 2, e = q & 3;
          const uint32_t p = wbase + bytes_before(tw, i) + byte_of(sl, i) +
                             static_cast<uint32_t>(__popc(f & ((1u << q) - 1u) & (0xFu << (4 * i))));
          const int pos = key_pos(i, e);
          put(p, float_order_key(staged[pos]), pos);
        }
      } else {
#pragma unroll
        for (int i = 0; i < kSteps; ++i) {
          uint32_t p = wbase + bytes_before(tw, i) + byte_of(sl, i);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int q = 4 * i + e;
            if ((f >> q) & 1u) {
              put(p, key[q], key_pos(i, e));
              ++p;
            }
          }
        }
      }
      // (the next chunk writes wsum only after its first barrier, which every
      // warp reaches after these reads)
    }
    own = min(own, static_cast<uint32_t>(kListCap));
    __syncthreads();
    auto entry_index = [&](uint32_t en) -> int {
      return (chunk0 + static_cast<int>((en >> 13) & 0x3Fu)) * kChunk + static_cast<int>(en & kOffMask);
    };
    // the order key of the row's key s (s < n), read again: staged, from the
    // slice while the list (entries [0, own)) has not reached its word
    auto key_again = [&](int s_idx) -> uint32_t {
      if (kStaged && kChunk + (s_idx - chunk0 * kChunk) >= static_cast<int>(own))
        return float_order_key(staged[s_idx]);
      return float_order_key(__ldg(row + s_idx));
    };

    // ---- 3. second digit: the row's counts in the leader
    if (C > 1) {
      wait_zeroed();
      const uint32_t l2 = map_rank(sm.h2, 0);
      for (int i = tid; i < kBins1; i += kThreads)
        if (sm.lh2[i]) red_add_cluster(l2 + 4u * i, sm.lh2[i]);
      cluster_sync();
    }
    const uint32_t rem1 = static_cast<uint32_t>(k) - above1;
    {
      const uint4 v = ld_cluster_v4(map_rank(sm.h2, 0) + 4u * (kBins1 - 4 - 4 * tid));
      uint32_t h[4] = {v.w, v.z, v.y, v.x};
      select_bin<4>(h, rem1, sm.wsum, &sm.res[3]);
    }
    const uint32_t D2 = sm.res[3];
    if (D2 == kNoBin) {
      give_up();
      leave();
      return;
    }
    const uint32_t rem2 = rem1 - sm.res[4];
    const uint32_t nb = sm.res[5];  // the row's keys in bin D2: the boundary
    uint32_t D3 = 0, take_eq = 0, gt_off = 0, eq_off = 0;
    bool offsets_known = false;
    if (nb <= static_cast<uint32_t>(kBndCap)) {
      // ---- 3'. few boundary keys: they travel with the counts.  Each CTA
      // publishes its boundary keys (read again for their full key) and its
      // count of keys certainly kept (sure, or second digit > D2); every CTA
      // then finds T among the row's boundary keys, the ties it keeps (lowest
      // index first), and its own output offset, with no further barrier.
      uint32_t gd = 0;
      const uint32_t lbnd = map_rank(sm.bnd, 0) + 8u * (c * kBndCap);
      for (uint32_t i = tid; i < own; i += kThreads) {
        const uint32_t en = sm.ent[i];
        const uint32_t d = (en >> 19) & 0x7FFu;
        if ((en & kSure) || d > D2) {
          ++gd;
        } else if (d == D2) {
          const uint32_t j = atomicAdd(&sm.bcount, 1u);
          const int s_idx = entry_index(en);
          const uint32_t kk = s_idx < n ? key_again(s_idx) : 0u;
          if (j < static_cast<uint32_t>(kBndCap)) {
            sm.bslot[j] = i;
            st_cluster(lbnd + 8u * j, kk);
            st_cluster(lbnd + 8u * j + 4u, static_cast<uint32_t>(s_idx));
          }
        }
      }
      gd = __reduce_add_sync(0xffffffffu, gd);
      if (lane == 0 && gd) atomicAdd(&sm.gdsum, gd);
      __syncthreads();
      const uint32_t my_nb = min(sm.bcount, static_cast<uint32_t>(kBndCap));
      if (tid == 0) st_cluster(map_rank(sm.kept, 0) + 4u * c, (sm.gdsum << 16) | my_nb);
      if (C > 1) cluster_sync();
      else __syncthreads();
      // every CTA's counts and boundary keys
      const uint32_t x = lane < C ? ld_cluster(map_rank(sm.kept, 0) + 4u * lane) : 0u;
      const uint32_t xb = x & 0xFFFFu, xi = warp_incl_scan(xb);
      const uint32_t nb_all = __shfl_sync(0xffffffffu, xi, 31);
      if (nb_all != nb) {  // (the counts do not add up: a mismatched histogram)
        give_up();
        leave();
        return;
      }
      if (warp == 0) {  // gather: lane l < C copies CTA l's boundary keys
        if (lane < C) {
          sm.bpre[lane] = xi - xb;
          const uint32_t src = map_rank(sm.bnd, 0) + 8u * (lane * kBndCap);
          for (uint32_t j = 0; j < xb; ++j)
            sm.bk[xi - xb + j] = make_uint2(ld_cluster(src + 8u * j), ld_cluster(src + 8u * j + 4u));
        }
      }
      __syncthreads();
      // T: the rem2-th largest boundary key
      if (tid < nb) {
        const uint32_t kt = sm.bk[tid].x;
        uint32_t gt = 0, eq = 0;
        for (uint32_t j = 0; j < nb; ++j) {
          gt += sm.bk[j].x > kt ? 1u : 0u;
          eq += sm.bk[j].x == kt ? 1u : 0u;
        }
        if (gt < rem2 && rem2 <= gt + eq) {
          sm.res[6] = kt;
          sm.res[7] = rem2 - gt;  // keys == T kept
          sm.found = 1;
        }
      }
      __syncthreads();
      if (!sm.found) {
        give_up();
        leave();
        return;
      }
      const uint32_t T = sm.res[6], keep_eq = sm.res[7];
      // which boundary keys are kept (ties: the lowest indices); each CTA's
      // kept count, and this CTA's own boundary entries rewritten as sure or
      // dropped (an entry with second digit 0 and no flags is never kept)
      if (tid < nb) {
        const uint2 e = sm.bk[tid];
        bool kept = e.x > T;
        if (e.x == T) {
          uint32_t rank = 0;
          for (uint32_t j = 0; j < nb; ++j) rank += (sm.bk[j].x == T && sm.bk[j].y < e.y) ? 1u : 0u;
          kept = rank < keep_eq;
        }
        int cc = 0;  // the CTA whose keys slot tid holds
        while (cc + 1 < C && sm.bpre[cc + 1] <= tid) ++cc;
        if (kept) atomicAdd(&sm.kbc[cc], 1u);
        if (cc == static_cast<int>(c)) {
          const uint32_t slot = sm.bslot[tid - sm.bpre[cc]];
          sm.ent[slot] = (kept ? kSure : 0u) | (sm.ent[slot] & kPosMask);
        }
      }
      __syncthreads();
      // this CTA's output offset: the kept keys of the lower-ranked CTAs
      {
        const uint32_t kept_l = lane < C ? (x >> 16) + sm.kbc[lane] : 0u;
        const uint32_t ki = warp_incl_scan(kept_l);
        gt_off = __shfl_sync(0xffffffffu, ki - kept_l, static_cast<int>(c));
        if (__shfl_sync(0xffffffffu, ki, 31) != static_cast<uint32_t>(k)) {
          give_up();
          leave();
          return;
        }
      }
      offsets_known = true;
    } else {
      // third digit of this CTA's entries in bin D2 (their keys are read
      // again), kept in place of their second digit; the row's counts in the
      // leader
      uint32_t* my_h3 = C > 1 ? sm.lh3 : sm.h3;
      for (uint32_t i = tid; i < own; i += kThreads) {
        const uint32_t en = sm.ent[i];
        if (!(en & kSure) && ((en >> 19) & 0x7FFu) == D2) {
          const int s_idx = entry_index(en);
          const uint32_t d3 = s_idx < n ? key_again(s_idx) & 0x3FFu : 0u;
          atomicAdd(&my_h3[d3], 1u);
          sm.ent[i] = kHasD3 | (d3 << 19) | (en & kPosMask);
        }
      }
      __syncthreads();
      if (C > 1) {
        const uint32_t l3 = map_rank(sm.h3, 0);
        for (int i = tid; i < kBins3; i += kThreads)
          if (sm.lh3[i]) red_add_cluster(l3 + 4u * i, sm.lh3[i]);
        cluster_sync();
      }
      {
        const uint32_t l3 = map_rank(sm.h3, 0);
        const uint2 v = make_uint2(ld_cluster(l3 + 4u * (kBins3 - 2 - 2 * tid)), ld_cluster(l3 + 4u * (kBins3 - 1 - 2 * tid)));
        uint32_t h[2] = {v.y, v.x};
        select_bin<2>(h, rem2, sm.wsum, &sm.res[6]);
      }
      D3 = sm.res[6];
      if (D3 == kNoBin) {
        give_up();
        leave();
        return;
      }
      take_eq = rem2 - sm.res[7];  // keys == T to keep, lowest index first
    }
    // ---- 4. kept keys: key > T, or key == T among the row's first take_eq of
    // them.  This CTA's list, in index order, by warps taking G entries each;
    // a kept key's output slot is the row's keys > T before it plus min(keys
    // == T before it, take_eq).
    auto classify = [&](uint32_t en) -> uint32_t {  // 2: key > T, 1: key == T, 0: below
      if (en & kSure) return 2u;
      const uint32_t d = (en >> 19) & 0x7FFu;
      if (en & kHasD3) return d > D3 ? 2u : (d == D3 ? 1u : 0u);
      return d > D2 ? 2u : 0u;  // (entries in bin D2 all carry their third digit)
    };
    const uint32_t G = (own + 32 * kWarps - 1) / (32 * kWarps) * 32;
    const uint32_t g_lo = static_cast<uint32_t>(warp) * G, g_hi = min(g_lo + G, own);
    {
      uint32_t g = 0, e = 0;
      for (uint32_t g0 = g_lo; g0 < g_hi; g0 += 32) {
        const uint32_t gg = g0 + lane;
        const uint32_t cl = gg < g_hi ? classify(sm.ent[gg]) : 0u;
        g += __popc(__ballot_sync(0xffffffffu, cl == 2u));
        e += __popc(__ballot_sync(0xffffffffu, cl == 1u));
      }
      if (lane == 0) sm.wcnt[warp] = (g << 16) | e;
    }
    __syncthreads();
    const uint32_t wc = lane < kWarps ? sm.wcnt[lane] : 0u;
    const uint32_t wi = warp_incl_scan(wc);
    const uint32_t mine = __shfl_sync(0xffffffffu, wi, 31);  // this CTA's keys > T, == T
    uint32_t row_gt = mine >> 16, row_eq = mine & 0xFFFFu;
    if (offsets_known) {
      row_gt = static_cast<uint32_t>(k);  // (checked with the boundary counts)
      row_eq = 0;
    } else if (C > 1) {
      // every CTA's counts through the leader: offsets from the lower ranks
      const uint32_t lk = map_rank(sm.kept, 0);
      if (tid == 0) st_cluster(lk + 4u * c, mine);
      cluster_sync();
      const uint32_t x = lane < C ? ld_cluster(lk + 4u * lane) : 0u;
      const uint32_t xlo = lane < static_cast<int>(c) ? x : 0u;
      uint32_t gs = x >> 16, es = x & 0xFFFFu, gl = xlo >> 16, el = xlo & 0xFFFFu;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        gs += __shfl_xor_sync(0xffffffffu, gs, off);
        es += __shfl_xor_sync(0xffffffffu, es, off);
        gl += __shfl_xor_sync(0xffffffffu, gl, off);
        el += __shfl_xor_sync(0xffffffffu, el, off);
      }
      row_gt = gs;
      row_eq = es;
      gt_off = gl;
      eq_off = el;
    }
    if (row_gt + min(row_eq, take_eq) != static_cast<uint32_t>(k)) {
      give_up();
      leave();
      return;
    }
    {
      const uint32_t before = __shfl_sync(0xffffffffu, wi - wc, warp);  // earlier warps of this CTA
      uint32_t gb = gt_off + (before >> 16), eb = eq_off + (before & 0xFFFFu);
      const uint32_t lt = lanemask_lt();
      for (uint32_t g0 = g_lo; g0 < g_hi; g0 += 32) {
        const uint32_t gg = g0 + lane;
        uint32_t cl = 0, s_idx = 0;
        if (gg < g_hi) {
          const uint32_t en = sm.ent[gg];
          cl = classify(en);
          s_idx = static_cast<uint32_t>(entry_index(en));
        }
        const uint32_t bg = __ballot_sync(0xffffffffu, cl == 2u), be = __ballot_sync(0xffffffffu, cl == 1u);
        const uint32_t g_before = gb + __popc(bg & lt), e_before = eb + __popc(be & lt);
        // (with a remap the key's list slot is written here and mapped below)
        if (cl == 2u) out[g_before + min(e_before, take_eq)] = static_cast<int32_t>(s_idx);
        else if (cl == 1u && e_before < take_eq) out[g_before + e_before] = static_cast<int32_t>(s_idx);
        gb += __popc(bg);
        eb += __popc(be);
      }
    }
    if (remap != nullptr) {
      // this CTA's kept keys fill the output slots [lo, hi)
      __syncthreads();  // (this CTA's writes of out are visible to all its threads)
      const uint32_t lo = gt_off + min(eq_off, take_eq);
      const uint32_t hi = gt_off + (mine >> 16) + min(eq_off + (mine & 0xFFFFu), take_eq);
      for (uint32_t j = lo + tid; j < hi; j += kThreads) out[j] = __ldg(remap + out[j]);
    }
    leave();
    return;
  }

  // ---- overflow (C == 1: one CTA walking a row whose listed keys exceed its
  // list): the second and third digits from histograms of the row's keys,
  // then the kept keys written chunk by chunk at running offsets
  for (int i = tid; i < kBins1; i += kThreads) sm.hist[i] = 0;
  __syncthreads();
  prefetch_chunk(1);
  for (int ch = 0; ch < nch; ++ch) {
    prefetch_chunk(ch + 2);
    chunk(ch);
    vm = load_slice(key);
#pragma unroll
    for (int q = 0; q < kPer; ++q)
      if (((vm >> q) & 1u) && (key[q] >> 21) == D1) atomicAdd(&sm.hist[(key[q] >> 10) & 0x7FFu], 1u);
  }
  __syncthreads();
  const uint32_t rem1 = static_cast<uint32_t>(k) - above1;
  {
    uint32_t h[4];
    my_bins4(sm.hist, h);
    select_bin<4>(h, rem1, sm.wsum, &sm.res[3]);
  }
  if (sm.res[3] == kNoBin) {
    give_up();
    pdl_trigger();
    return;
  }
  const uint32_t pref22 = (D1 << 11) | sm.res[3];
  const uint32_t rem2 = rem1 - sm.res[4];
  for (int i = tid; i < kBins1; i += kThreads) sm.hist[i] = 0;
  __syncthreads();
  prefetch_chunk(1);
  for (int ch = 0; ch < nch; ++ch) {
    prefetch_chunk(ch + 2);
    chunk(ch);
    vm = load_slice(key);
#pragma unroll
    for (int q = 0; q < kPer; ++q)
      if (((vm >> q) & 1u) && (key[q] >> 10) == pref22) atomicAdd(&sm.hist[key[q] & 0x3FFu], 1u);
  }
  __syncthreads();
  {
    uint32_t h[2];
    my_bins2(sm.hist, h);
    select_bin<2>(h, rem2, sm.wsum, &sm.res[6]);
  }
  if (sm.res[6] == kNoBin) {
    give_up();
    pdl_trigger();
    return;
  }
  const uint32_t T = (pref22 << 10) | sm.res[6];
  const uint32_t take_eq = rem2 - sm.res[7];
  pdl_trigger();
  uint32_t gt_off = 0, eq_off = 0;
  prefetch_chunk(1);
  for (int ch = 0; ch < nch; ++ch) {
    prefetch_chunk(ch + 2);
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
  if (tid == 0 && gt_off + min(eq_off, take_eq) != static_cast<uint32_t>(k)) raise_error(P.err, kErrHistMismatch);
}

}  // namespace

size_t topk_workspace_bytes(int, int, int, int) { return 0; }

namespace {
// Launch one instance (cluster dimension C) with PDL; its attributes are set
// once per device.
template <int kCtaChunks, int kListCap, int kMinBlocks>
dsa_status_t launch_topk(const RowSel& P, int64_t rows, int C, int device, cudaStream_t stream) {
  auto kern = topk_cluster_kernel<kCtaChunks, kListCap, kMinBlocks>;
  constexpr int kEntWords = kMinBlocks == 1 ? kCtaChunks * kChunk + kChunk : kListCap;  // as in the kernel
  constexpr int kBndCtas = kMinBlocks == 1 ? kMaxCluster : 1;
  const size_t smem = sizeof(TopkSmem<kEntWords, kBndCtas>);
  static_assert(kMinBlocks == 1 || 2 * (sizeof(TopkSmem<kEntWords, kBndCtas>) + 1024) <= 233472,
                "two CTAs an SM");
  static bool attr_done[64] = {};
  if (device < 0 || device >= 64) return DSA_ERR_UNSUPPORTED;
  if (!attr_done[device]) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) !=
            cudaSuccess ||
        cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess)
      return DSA_ERR_CUDA;
    attr_done[device] = true;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(rows * C), 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = static_cast<unsigned>(C);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1] = pdl_attribute();
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, kern, P) == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}
}  // namespace

dsa_status_t topk_radix(const TopkArgs& a) {
  const int64_t rows = static_cast<int64_t>(a.B) * a.n_q;
  if (rows == 0) return DSA_OK;
  static_assert(kClusterSlice < 65536 && kListCapCluster < 65536 && kListCapRow < 65536,
                "per-warp and per-CTA counts are packed in 16 bits");
  static_assert(kClusterSlice <= kListCapCluster, "a CTA of a cluster lists at most its slice");
  static_assert(kMaxCluster <= 32, "per-CTA counts summed by one warp");
  static_assert(kMaxCluster * kClusterChunks <= 64, "a walking CTA's chunk fits the entry's 6-bit field");
  const int64_t n_max = std::max(1, a.s_max);
  if (n_max > static_cast<int64_t>(kMaxCluster) * kClusterSlice) return DSA_ERR_UNSUPPORTED;
  int64_t C = (n_max + kClusterSlice - 1) / kClusterSlice;
  // many rows (prefill rounds): a CTA a row, walking it in chunks, so that
  // many rows are in flight; few long rows (decode): a cluster a row
  if (rows >= 2LL * std::max(1, device_sm_count(a.device))) C = 1;
  if (rows * C > INT32_MAX) return DSA_ERR_UNSUPPORTED;
  if (a.k <= 0) return DSA_ERR_INVALID_ARG;
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
  P.err = a.err;
  if (P.hist_parts != nullptr && (P.hist_per_cta <= 0 || P.hist_tpr <= 0)) return DSA_ERR_INVALID_ARG;
  if (P.hist_parts != nullptr && (reinterpret_cast<uintptr_t>(P.hist_parts) & 15u) != 0) return DSA_ERR_INVALID_ARG;
  // one CTA a row: few rows that fit a staged slice (short decode contexts,
  // candidate lists) take the staged instance, many rows walk theirs
  if (C == 1 && rows < 2LL * std::max(1, device_sm_count(a.device)) && n_max <= kClusterSlice)
    return launch_topk<kClusterChunks, kListCapCluster, 1>(P, rows, 1, a.device, a.stream);
  if (C == 1) return launch_topk<kClusterChunks, kListCapRow, 2>(P, rows, 1, a.device, a.stream);
  return launch_topk<kClusterChunks, kListCapCluster, 1>(P, rows, static_cast<int>(C), a.device, a.stream);
}

}  // namespace dsa
