// Fine-grained token selection: per query, the index_topk best-scored
// previous keys (DeepSeek-V3.2 model doc, Transformers, section "DeepSeek
// Sparse Attention (DSA)", item 2; index_topk defaults to 2048).
//
// Radix select on order-preserving 32-bit keys, no sort, one CTA per query
// row.  The key splits into digits of 11, 11 and 10 bits (most significant
// first); T, the key of the k-th largest score, is found digit by digit:
//   1. histogram of the first digit over the row (or the sum of the partial
//      histograms the indexer's epilogue built, see TopkArgs::hist_parts),
//      then the bin D1 that holds the k-th largest key;
//   2. one pass over the row that keeps, in index order, the "sure" keys
//      (first digit > D1: fewer than k of them) and the candidates (first
//      digit == D1: on index scores a few thousand out of 128K) in shared
//      memory, with the histogram of the candidates' second digit;
//   3. the third digit from the candidates held in shared memory, then the
//      output: the sure keys and the selected candidates (key > T, plus the
//      lowest-indexed keys == T: ties go to the lower index) are two
//      ascending lists, merged by binary search into ascending order.
// The row streams through a two-stage shared-memory ring filled by bulk
// copies (64 KB a chunk, two in flight), so a pass over a 128K-key row is
// bound by the copy rate, not by the loads a thread can keep in flight.
// Rows whose candidates do not fit the shared-memory lists (e.g. all scores
// equal) take the same digits from further passes over the row and finish
// with an ordered compaction pass.  Rows with at most k candidates are
// written directly.
#include "dsa_common.cuh"
#include "dsa_internal.h"

namespace dsa {
namespace {

constexpr int kBins1 = 2048;  // first and second digits: 11 bits
constexpr int kBins3 = 1024;  // third digit: 10 bits
constexpr int kMaxWarps = 32;
constexpr int kCandCap = 8192;     // candidates kept in shared memory, at most
constexpr int kSureCapMax = 4096;  // sure keys kept in shared memory (< k of them), at most

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
// *total.  Uses `wsum` (kMaxWarps + 1 words).  Ends with a barrier, so wsum
// may be reused at once.
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

// The bin of `hist` (nbins, counted from the top) that holds the
// `remaining`-th largest key: *digit, and *above = keys in higher bins.
template <int kThreads>
__device__ __forceinline__ void select_bin(const uint32_t* hist, int nbins, uint32_t remaining, uint32_t* wsum,
                                           uint32_t* s_digit, uint32_t* s_above) {
  const int bpt = nbins / kThreads;  // bins a thread, taken from the top
  const int top = nbins - 1 - static_cast<int>(threadIdx.x) * bpt;
  uint32_t cnt = 0;
  for (int i = 0; i < bpt; ++i) cnt += hist[top - i];
  uint32_t total;
  const uint32_t excl = block_excl_scan<kThreads>(cnt, wsum, &total);
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

// Bulk copy of `bytes` (a multiple of 16) from global memory into this CTA's
// shared memory, completing on `bar` (this CTA only).
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "l"(src), "r"(bytes), "r"(bar)
               : "memory");
}

// The score row streamed through a two-stage shared-memory ring: chunk c of
// a pass (kChunk keys) lands in stage (g + c) & 1, where g counts the chunks
// of earlier passes; thread 0 issues the copies two chunks ahead.  Every
// thread reads PER keys of the chunk from shared memory (layout at pos()).
template <int kThreads, int PER>
struct RowStream {
  static constexpr int kChunk = kThreads * PER;
  const float* row;
  int n, nchunks;
  uint32_t ring, bar;  // shared addresses: stage 0, full barrier of stage 0
  uint32_t g;          // chunks streamed by earlier passes
  uint32_t issued[2];  // copies issued into each stage (thread 0's count)
  uint32_t* err;
  volatile int* abort_flag;

  __device__ __forceinline__ uint32_t bytes(int c) const {
    const int keys = min(kChunk, n - c * kChunk);
    return static_cast<uint32_t>((keys + 3) & ~3) * 4u;  // whole 16-byte pieces (the row stride is one too)
  }
  __device__ __forceinline__ void issue(int c) {
    const uint32_t st = (g + c) & 1u;
    ++issued[st];
    mbar_arrive_expect_tx(bar + 8u * st, bytes(c));
    bulk_g2s(ring + st * (kChunk * 4u), row + static_cast<int64_t>(c) * kChunk, bytes(c), bar + 8u * st);
  }
  // Start a pass: the first two chunks in flight.
  __device__ __forceinline__ void begin() {
    if (threadIdx.x == 0) {
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // earlier reads of the ring come first
      for (int c = 0; c < 2 && c < nchunks; ++c) issue(c);
    }
  }
  // Key (i, e) of this thread in chunk c: warp w covers the chunk's keys
  // [w 32 PER, (w + 1) 32 PER); in step i its lane l holds the four keys
  // 4 (32 i + l) + e of that range, so a step's shared-memory reads are 16
  // consecutive bytes a lane (no bank conflicts) and the keys of a warp are
  // in index order (step, lane, element).
  __device__ __forceinline__ int pos(int c, int i, int e) const {
    return c * kChunk + (static_cast<int>(threadIdx.x) >> 5) * (32 * PER) + 4 * (32 * i + lane_id()) + e;
  }
  // Wait for chunk c and load this thread's keys (key[4 i + e]); false on a
  // wait that expired.
  __device__ __forceinline__ bool load(int c, uint32_t* key, uint32_t* vmask) const {
    const uint32_t gg = g + c;
    if (!mbar_wait_warp(bar + 8u * (gg & 1u), (gg >> 1) & 1u, abort_flag, err)) return false;
    const uint32_t src = ring + (gg & 1u) * (kChunk * 4u) + (threadIdx.x >> 5) * (32u * PER * 4u) + lane_id() * 16u;
    uint32_t vm = 0;
#pragma unroll
    for (int i = 0; i < PER / 4; ++i) {
      float4 f;
      asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
                   : "=f"(f.x), "=f"(f.y), "=f"(f.z), "=f"(f.w)
                   : "r"(src + i * 512u)
                   : "memory");
      key[4 * i] = float_order_key(f.x);
      key[4 * i + 1] = float_order_key(f.y);
      key[4 * i + 2] = float_order_key(f.z);
      key[4 * i + 3] = float_order_key(f.w);
      const int p0 = pos(c, i, 0);
#pragma unroll
      for (int e = 0; e < 4; ++e) vm |= (p0 + e < n ? 1u : 0u) << (4 * i + e);
    }
    *vmask = vm;
    return true;
  }
  // Every thread is done with chunk c (call after a barrier): refill its
  // stage with chunk c + 2.
  __device__ __forceinline__ void release(int c) {
    if (threadIdx.x == 0 && c + 2 < nchunks) {
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      issue(c + 2);
    }
  }
  __device__ __forceinline__ void end() { g += nchunks; }
  // After a wait that expired: let the copies still in flight land (bounded)
  // before the shared memory is released.
  __device__ __forceinline__ void drain() const {
    if (threadIdx.x == 0) {
      volatile int never = 0;
      for (uint32_t st = 0; st < 2; ++st)
        if (issued[st] > 0) mbar_wait(bar + 8u * st, (issued[st] - 1u) & 1u, &never, err);
    }
    __syncthreads();
  }
};

// Index-order offsets of this thread's flagged keys for two flag sets a and
// b (bit 4 i + e = key (i, e) of RowStream's layout): offa[i] (offb[i]) =
// flagged keys of the block's chunk before this thread's step-i keys, taking
// the warps in order, then steps, then lanes.  Returns the chunk's totals
// (a << 16 | b).  One packed warp scan (four 8-bit step counts) per set and
// one block scan over the warps' totals.
template <int kThreads, int PER>
__device__ __forceinline__ uint32_t ordered_offsets(uint32_t fa, uint32_t fb, uint32_t* offa, uint32_t* offb,
                                                    uint32_t* wsum) {
  static_assert(PER == 16, "four steps of four keys a lane");
  constexpr int kWarps = kThreads / 32;
  const int lane = lane_id(), warp = threadIdx.x >> 5;
  uint32_t ca = 0, cb = 0;  // this lane's count per step, one byte each
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    ca |= static_cast<uint32_t>(__popc((fa >> (4 * i)) & 0xFu)) << (8 * i);
    cb |= static_cast<uint32_t>(__popc((fb >> (4 * i)) & 0xFu)) << (8 * i);
  }
  const uint32_t ia = warp_incl_scan(ca), ib = warp_incl_scan(cb);
  const uint32_t ta = __shfl_sync(0xffffffffu, ia, 31), tb = __shfl_sync(0xffffffffu, ib, 31);  // step totals
  const uint32_t ea = ia - ca, eb = ib - cb;
  uint32_t wa = 0, wb = 0;  // warp totals
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    offa[i] = wa + ((ea >> (8 * i)) & 0xFFu);
    offb[i] = wb + ((eb >> (8 * i)) & 0xFFu);
    wa += (ta >> (8 * i)) & 0xFFu;
    wb += (tb >> (8 * i)) & 0xFFu;
  }
  if (lane == 0) wsum[warp] = (wa << 16) | wb;
  __syncthreads();
  if (warp == 0) {
    const uint32_t x = lane < kWarps ? wsum[lane] : 0u;
    const uint32_t xi = warp_incl_scan(x);
    if (lane < kWarps) wsum[lane] = xi - x;
    if (lane == 31) wsum[kWarps] = xi;
  }
  __syncthreads();
  const uint32_t base = wsum[warp];
  const uint32_t total = wsum[kWarps];
  __syncthreads();
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    offa[i] += base >> 16;
    offb[i] += base & 0xFFFFu;
  }
  return total;
}

struct RowSel {
  const float* scores;
  int64_t ld;
  const int32_t* ctx_len;
  const int32_t* q_pos0;
  int t_off, n_q, s_max, k;
  int32_t* idx;
  const int32_t* remap;        // output idx = remap[row * remap_ld + s] (or s when null)
  int64_t remap_ld;
  const uint32_t* hist_parts;  // the indexer's partial first-digit histograms, or null
  int hist_per_cta, hist_tpr;
  int sure_cap, cand_cap;      // shared-memory list sizes (entries; cand_cap a multiple of the block size)
  uint32_t* err;
};

template <int kThreads, int PER>
__global__ void __launch_bounds__(kThreads, 1) topk_row_kernel(RowSel P) {
  pdl_wait();
  using Stream = RowStream<kThreads, PER>;
  constexpr int kChunk = Stream::kChunk;
  constexpr int kFixedWords = 2 * kChunk + 2 * kBins1 + kBins3 + 64 + 8;
  extern __shared__ __align__(128) uint32_t sm[];
  float* ring = reinterpret_cast<float*>(sm);  // [2][kChunk]
  uint32_t* hist1 = sm + 2 * kChunk;           // [2048]
  uint32_t* hist2 = hist1 + kBins1;            // [2048]
  uint32_t* hist3 = hist2 + kBins1;            // [1024]
  uint32_t* wsum = hist3 + kBins3;             // [kMaxWarps + 1], then 8 words of results
  uint32_t* res = wsum + kMaxWarps + 1;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + 2 * kChunk + 2 * kBins1 + kBins3 + 64);  // [2]: full barriers
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 2);
  int32_t* sure = reinterpret_cast<int32_t*>(sm + kFixedWords);    // [sure_cap]
  int32_t* selc = sure + P.sure_cap;                                 // [sure_cap]
  uint32_t* ckey = reinterpret_cast<uint32_t*>(selc + P.sure_cap);  // [cand_cap]
  int32_t* cidx = reinterpret_cast<int32_t*>(ckey + P.cand_cap);    // [cand_cap]

  const int r = blockIdx.x;
  const int b = r / P.n_q, t = r % P.n_q;
  const int L = min(max(__ldg(P.ctx_len + b), 0), P.s_max);
  const int n = max(0, min(__ldg(P.q_pos0 + b) + P.t_off + t + 1, L));  // candidates s in [0, n)
  int32_t* out = P.idx + static_cast<int64_t>(r) * P.k;
  const int32_t* remap = P.remap ? P.remap + static_cast<int64_t>(r) * P.remap_ld : nullptr;
  const int tid = threadIdx.x;
  auto emit = [&](int pos, int s) { out[pos] = remap ? __ldg(remap + s) : s; };

  if (n <= P.k) {
    for (int j = tid; j < P.k; j += kThreads) {
      if (j < n) emit(j, j);
      else out[j] = -1;
    }
    pdl_trigger();
    return;
  }

  Stream S;
  S.row = P.scores + static_cast<int64_t>(r) * P.ld;
  S.n = n;
  S.nchunks = (n + kChunk - 1) / kChunk;
  S.ring = smem_addr(ring);
  S.bar = smem_addr(bars);
  S.g = 0;
  S.issued[0] = S.issued[1] = 0;
  S.err = P.err;
  S.abort_flag = abort_flag;
  if (tid == 0) {
    mbar_init(S.bar, 1);
    mbar_init(S.bar + 8, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  for (int i = tid; i < 2 * kBins1 + kBins3; i += kThreads) hist1[i] = 0;
  __syncthreads();

  // ---- 1. first digit
  if (P.hist_parts != nullptr) {
    // row r's key tiles [r tpr, (r + 1) tpr) were scored by the indexer CTAs
    // c_lo..c_hi (runs of per_cta tiles); CTA c kept this row in slot 0 if
    // its run starts in it, else in slot 1
    const int64_t tile0 = static_cast<int64_t>(r) * P.hist_tpr;
    const int c_lo = static_cast<int>(tile0 / P.hist_per_cta);
    const int c_hi = static_cast<int>((tile0 + P.hist_tpr - 1) / P.hist_per_cta);
    S.begin();  // the candidate pass's first chunks load under the histogram sum
    for (int i = tid; i < kBins1; i += kThreads) {
      uint32_t v = 0;
      for (int c = c_lo; c <= c_hi; ++c) {
        const int slot = (static_cast<int64_t>(c) * P.hist_per_cta) / P.hist_tpr == r ? 0 : 1;
        v += __ldg(P.hist_parts + (static_cast<int64_t>(c) * 2 + slot) * kBins1 + i);
      }
      hist1[i] = v;
    }
  } else {
    S.begin();
    for (int c = 0; c < S.nchunks; ++c) {
      uint32_t key[PER], vm = 0;
      const bool ok = S.load(c, key, &vm);
#pragma unroll
      for (int e = 0; e < PER; ++e)
        if (ok && ((vm >> e) & 1u)) atomicAdd(&hist1[key[e] >> 21], 1u);
      if (__syncthreads_or(!ok)) {
        S.drain();
        return;
      }
      S.release(c);
    }
    S.end();
    S.begin();
  }
  __syncthreads();
  select_bin<kThreads>(hist1, kBins1, static_cast<uint32_t>(P.k), wsum, &res[0], &res[1]);
  const uint32_t D1 = res[0];
  const uint32_t above1 = res[1];  // sure keys (first digit > D1)
  const uint32_t ncand = hist1[D1];
  const bool fits = ncand <= static_cast<uint32_t>(P.cand_cap) && above1 <= static_cast<uint32_t>(P.sure_cap) &&
                    static_cast<uint32_t>(P.k) - above1 <= static_cast<uint32_t>(P.sure_cap);

  // ---- 2. sure keys and candidates, second digit (one pass, already started)
  {
    uint32_t sure_base = 0, cand_base = 0;
    for (int c = 0; c < S.nchunks; ++c) {
      uint32_t key[PER], vm = 0;
      const bool ok = S.load(c, key, &vm);
      uint32_t fs = 0, fc = 0;  // sure / candidate flags, bit 4 i + e
#pragma unroll
      for (int e = 0; e < PER; ++e) {
        const bool v = ok && ((vm >> e) & 1u);
        const uint32_t d = key[e] >> 21;
        fs |= (v && d > D1) ? (1u << e) : 0u;
        if (v && d == D1) {
          fc |= 1u << e;
          atomicAdd(&hist2[(key[e] >> 10) & 0x7FFu], 1u);
        }
      }
      if (fits) {
        uint32_t os[4], oc[4];
        const uint32_t tot = ordered_offsets<kThreads, PER>(fs, fc, os, oc, wsum);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          uint32_t ps = sure_base + os[i], pc = cand_base + oc[i];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int q = 4 * i + e;
            if ((fs >> q) & 1u) {
              sure[ps++] = S.pos(c, i, e);
            } else if ((fc >> q) & 1u) {
              ckey[pc] = key[q];
              cidx[pc] = S.pos(c, i, e);
              ++pc;
            }
          }
        }
        sure_base += tot >> 16;
        cand_base += tot & 0xFFFFu;
      }
      if (__syncthreads_or(!ok)) {
        S.drain();
        return;
      }
      S.release(c);
    }
    S.end();
  }
  __syncthreads();
  const uint32_t rem1 = static_cast<uint32_t>(P.k) - above1;
  select_bin<kThreads>(hist2, kBins1, rem1, wsum, &res[2], &res[3]);
  const uint32_t D2 = res[2];
  const uint32_t rem2 = rem1 - res[3];
  const uint32_t pref22 = (D1 << 11) | D2;  // the key's top 22 bits at T

  // ---- 3. third digit
  if (fits) {
    for (uint32_t i = tid; i < ncand; i += kThreads) {
      const uint32_t kk = ckey[i];
      if ((kk >> 10) == pref22) atomicAdd(&hist3[kk & 0x3FFu], 1u);
    }
  } else {
    S.begin();
    for (int c = 0; c < S.nchunks; ++c) {
      uint32_t key[PER], vm = 0;
      const bool ok = S.load(c, key, &vm);
#pragma unroll
      for (int e = 0; e < PER; ++e)
        if (ok && ((vm >> e) & 1u) && (key[e] >> 10) == pref22) atomicAdd(&hist3[key[e] & 0x3FFu], 1u);
      if (__syncthreads_or(!ok)) {
        S.drain();
        return;
      }
      S.release(c);
    }
    S.end();
  }
  __syncthreads();
  select_bin<kThreads>(hist3, kBins3, rem2, wsum, &res[4], &res[5]);
  const uint32_t T = (pref22 << 10) | res[4];
  const uint32_t take_eq = rem2 - res[5];  // keys == T to keep, lowest index first
  pdl_trigger();                           // the selection is fixed; only the writes remain

  if (fits) {
    // selected candidates (ascending, since the list is in index order):
    // key > T, or key == T among the first take_eq of them
    const int cpt = P.cand_cap / kThreads;  // candidates a thread, consecutive
    const int c0 = tid * cpt;
    uint32_t gt = 0, eq = 0;
    for (int e = 0; e < cpt; ++e) {
      const int i = c0 + e;
      if (i < static_cast<int>(ncand)) {
        gt += ckey[i] > T ? 1u : 0u;
        eq += ckey[i] == T ? 1u : 0u;
      }
    }
    uint32_t tot;
    const uint32_t pre = block_excl_scan<kThreads>((gt << 16) | eq, wsum, &tot);
    uint32_t eq_rank = pre & 0xFFFFu;
    uint32_t pos = (pre >> 16) + min(eq_rank, take_eq);
    for (int e = 0; e < cpt; ++e) {
      const int i = c0 + e;
      if (i >= static_cast<int>(ncand)) break;
      const uint32_t kk = ckey[i];
      if (kk > T) {
        selc[pos++] = cidx[i];
      } else if (kk == T) {
        if (eq_rank < take_eq) selc[pos++] = cidx[i];
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
      const int sv = from_sure ? sure[j] : selc[j];
      const int32_t* other = from_sure ? selc : sure;
      int lo = 0, hi = from_sure ? n_sel : n_sure;  // count of `other` entries < sv
      while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (other[mid] < sv) lo = mid + 1;
        else hi = mid;
      }
      emit(j + lo, sv);
    }
  } else {
    // ordered compaction over the row: keys > T, and keys == T while fewer
    // than take_eq have been kept
    uint32_t gt_base = 0, eq_base = 0;
    S.begin();
    for (int c = 0; c < S.nchunks; ++c) {
      uint32_t key[PER], vm = 0;
      const bool ok = S.load(c, key, &vm);
      uint32_t fg = 0, fe = 0;  // key > T / key == T flags, bit 4 i + e
#pragma unroll
      for (int e = 0; e < PER; ++e) {
        const bool v = ok && ((vm >> e) & 1u);
        fg |= (v && key[e] > T) ? (1u << e) : 0u;
        fe |= (v && key[e] == T) ? (1u << e) : 0u;
      }
      uint32_t og[4], oe[4];
      const uint32_t tot = ordered_offsets<kThreads, PER>(fg, fe, og, oe, wsum);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        uint32_t gtc = gt_base + og[i], eqc = eq_base + oe[i];  // keys > T / == T before this one
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int q = 4 * i + e;
          if ((fg >> q) & 1u) {
            emit(gtc + min(eqc, take_eq), S.pos(c, i, e));
            ++gtc;
          } else if ((fe >> q) & 1u) {
            if (eqc < take_eq) emit(gtc + eqc, S.pos(c, i, e));
            ++eqc;
          }
        }
      }
      gt_base += tot >> 16;
      eq_base += tot & 0xFFFFu;
      if (__syncthreads_or(!ok)) {
        S.drain();
        return;
      }
      S.release(c);
    }
    S.end();
  }
}

constexpr int kRowThreads = 1024;
constexpr int kRowPer = 16;
constexpr size_t kSmemLimit = 232448;

// Shared memory of the kernel: the ring, histograms, scan words and
// barriers (fixed), then the lists: sure and selected keys (sure_cap each),
// candidate keys and indices (cand_cap each).
size_t row_fixed_bytes() {
  return (2 * static_cast<size_t>(kRowThreads) * kRowPer + 2 * kBins1 + kBins3 + 64 + 8) * 4;
}

}  // namespace

size_t topk_workspace_bytes(int, int, int, int) { return 0; }

dsa_status_t topk_radix(const TopkArgs& a) {
  const int64_t rows = static_cast<int64_t>(a.B) * a.n_q;
  if (rows == 0) return DSA_OK;
  if (rows > INT32_MAX) return DSA_ERR_UNSUPPORTED;
  static_assert(kRowThreads * kRowPer < 65536, "per-chunk counts are packed in 16 bits");
  RowSel P;
  P.scores = a.scores;
  P.ld = a.ld;
  P.ctx_len = a.ctx_len;
  P.q_pos0 = a.q_pos0;
  P.t_off = a.t_off;
  P.n_q = a.n_q;
  P.s_max = a.s_max;
  P.k = a.k;
  P.idx = a.idx;
  P.remap = a.remap;
  P.remap_ld = a.remap_ld;
  P.hist_parts = a.hist_parts;
  P.hist_per_cta = a.hist_per_cta;
  P.hist_tpr = a.hist_tpr;
  P.err = a.err;
  if (P.hist_parts != nullptr && (P.hist_per_cta <= 0 || P.hist_tpr <= 0)) return DSA_ERR_INVALID_ARG;
  // bulk copies read whole 16-byte pieces of a row: rows start on them
  if ((reinterpret_cast<uintptr_t>(a.scores) & 15u) != 0 || (a.ld & 3) != 0) return DSA_ERR_INVALID_ARG;
  P.sure_cap = std::min(a.k, kSureCapMax);
  const size_t room = kSmemLimit - row_fixed_bytes() - 2 * static_cast<size_t>(P.sure_cap) * 4;
  P.cand_cap = static_cast<int>(std::min<size_t>(kCandCap, room / 8) / kRowThreads * kRowThreads);
  if (P.cand_cap < kRowThreads) return DSA_ERR_UNSUPPORTED;
  const size_t smem =
      row_fixed_bytes() + 2 * static_cast<size_t>(P.sure_cap) * 4 + static_cast<size_t>(P.cand_cap) * 8;
  auto kern = topk_row_kernel<kRowThreads, kRowPer>;
  static size_t attr_smem[64] = {};
  if (a.device < 0 || a.device >= 64) return DSA_ERR_UNSUPPORTED;
  if (attr_smem[a.device] < smem) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) !=
        cudaSuccess)
      return DSA_ERR_CUDA;
    attr_smem[a.device] = smem;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(rows), 1, 1);
  cfg.blockDim = dim3(kRowThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = a.stream;
  cudaLaunchAttribute attr[1] = {pdl_attribute()};
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, P) == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

}  // namespace dsa
