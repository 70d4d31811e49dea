// Sparse MLA attention over the selected latent rows, on the tensor cores.
//
// DeepSeek-V3.2 model doc (Transformers), section "DeepSeek Sparse Attention
// (DSA)", item 2: main MLA attention runs only over the index_topk tokens the
// indexer kept, O(index_topk) per query instead of O(L).  Absorbed (MQA) form
// of MLA (section DeepseekV32Config: num_attention_heads 128, kv_lora_rank
// 512, qk_rope_head_dim 64): every head's 576-wide query meets one shared
// 576-wide latent row per token; the value is the row's first 512 columns.
//
// One thread-block cluster of two CTAs per (query row, split of its selected
// list).  The 576 latent columns are cut at 256: CTA 0 owns columns [0, 256),
// CTA 1 owns [256, 576); CTA c also owns the softmax of heads [64c, 64c + 64).
// Per 64-row tile, each CTA
//   * gathers only its own columns of the selected rows (cp.async, 16 bytes a
//     thread, into a 3-stage ring in the 128-byte-swizzled K-major layout the
//     MMA reads; padding and out-of-range rows are zero filled),
//   * computes its partial logits S_c = Q_c K_c^T for all 128 heads (M = 128,
//     N = 64, Q_c held in tensor memory),
//   * reduce-scatter: ships the partial logits of the other CTA's 64 heads
//     (16 KB, one bulk copy into the other CTA's shared memory) and adds the
//     partial it receives for its own 64 heads, so each CTA holds the full
//     S = S_0 + S_1 for the heads whose softmax it runs,
//   * runs the online softmax of its 64 heads (base 2; the running max only
//     moves, and O is rescaled in TMEM, when a tile max exceeds it by more
//     than 8) and writes their P rows in bf16,
//   * all-gather: ships those P rows (8 KB) and the heads' running max and
//     partial sums to the other CTA, which rescales its O rows of those heads
//     when the max moved,
//   * accumulates its 256-column half of the output, O_c += P V_c, in TMEM
//     (V_0 = latent columns [0, 256), V_1 = [256, 512): each CTA's value half
//     lies inside the columns it already gathered).
// Exchange buffers, P and the row statistics are double buffered so that
// tile j's exchange overlaps tile j-1's softmax, and the softmax warps read
// tile j+1's logits before they wait for tile j's partial.
// Warps: 0-3 gather, 4 issues tcgen05.mma, 5-12 (two per TMEM lane quarter,
// thread = head = TMEM lane): in the quarters of this CTA's own heads both
// warps run the softmax, 32 of the tile's 64 columns each; in the other
// quarters one warp ships the partial logits and one applies the other CTA's
// P statistics to this CTA's O rows.  Long selections are split across
// clusters and merged by a small combine kernel (log-sum-exp weights).  Every
// wait is bounded.
#include "dsa_common.cuh"
#include "dsa_internal.h"

namespace dsa {
namespace {

constexpr int kH = 128;                  // heads == MMA M
constexpr int kHHalf = 64;               // heads whose softmax one CTA runs
constexpr int kDqk = 576;                // latent 512 + rope 64
constexpr int kDv = 512;
constexpr int kDvHalf = 256;
constexpr int kRows = 64;                // selected rows per tile (MMA N of S, K of PV)
constexpr int kSplitCol = 256;           // CTA 0: columns [0, 256); CTA 1: [256, 576)
constexpr int kAtomsMax = 5;             // 64-column swizzle atoms per CTA (CTA 0 uses 4)
constexpr int kAtomBytes = kRows * 128;  // one atom of one tile: 8 KB
constexpr int kStageBytes = kAtomsMax * kAtomBytes;  // 40 KB
constexpr int kStages = 3;
constexpr int kPrefetchAhead = 6;        // tiles whose rows are pulled into L2 ahead of their gather
constexpr int kGatherWarps = 4;
constexpr int kMmaWarp = 4;
constexpr int kSoftWarps = 8;
constexpr int kPrefetchWarp = kGatherWarps + 1 + kSoftWarps;    // 13
constexpr int kThreads = 32 * (kPrefetchWarp + 1);               // 448
// tensor memory: O half [0, 256), Q columns [256, 256 + 160), S [416, 480)
constexpr int kTmemCols = 512;
constexpr int kQCol = 256;
constexpr int kSCol = 416;

// shared memory map (from a 1024-aligned base); [2] = double buffered by tile parity
constexpr int kPBytes = kH * kRows * 2;      // P: 128 heads x 64 rows bf16, SW128 K-major
constexpr int kPHalfBytes = kPBytes / 2;     // the 64 rows of one CTA's heads (contiguous)
constexpr int kXBytes = kHHalf * kRows * 4;  // partial logits of 64 heads: [16 x 4 rows][64 heads] fp32
constexpr int kStatBytes = 3 * kHHalf * 4;   // per head: running max, partial sum of each softmax warp
constexpr int kOffKV = 0;
constexpr int kOffP = kOffKV + kStages * kStageBytes;
constexpr int kOffXin = kOffP + 2 * kPBytes;      // partial logits received for this CTA's heads
constexpr int kOffXout = kOffXin + 2 * kXBytes;   // partial logits of the other CTA's heads, to ship
constexpr int kOffStOut = kOffXout + 2 * kXBytes; // statistics of this CTA's heads, to ship
constexpr int kOffStIn = kOffStOut + 2 * kStatBytes;
constexpr int kOffRed = kOffStIn + 2 * kStatBytes;  // tile max of each softmax warp: [2][2 warps][64]
// barriers: kv_full[3], kv_empty[3], q_ready, s_full, s_empty, mma_done, fin,
// pside_done, then 11 double-buffered ones (see the enum in the kernel)
constexpr int kNumDBars = 11;
constexpr int kNumBars = 2 * kStages + 6 + 2 * kNumDBars;
constexpr int kOffBar = kOffRed + 2 * 2 * kHHalf * 4;
constexpr int kOffMisc = kOffBar + kNumBars * 8;
constexpr int kSmemBytes = kOffMisc + 16 + 1024;
static_assert(kSmemBytes <= 232448, "shared memory");
static_assert(kOffP % 1024 == 0 && kPBytes % 1024 == 0, "P tiles must stay 1024-aligned");

struct AttnParams {
  const uint16_t* q;        // [R][128][576] bf16
  const uint16_t* kv;       // [B][s_max][576] bf16
  const int32_t* idx;       // [R][k]
  const int32_t* ctx_len;   // [B]
  __nv_bfloat16* out;       // [R][128][512]
  float* lse;               // [R][128] or null
  float* part_o;            // [R][S][2][128][256] (splits > 1)
  float* part_ml;           // [R][S][2][128]: m then l (splits > 1)
  int n_q, s_max, k, splits, rows_per_split;
  float scale_log2;         // sm_scale * log2(e)
  uint32_t* err;
};

// Shared-memory descriptor with explicit offsets and swizzle mode.
__device__ __forceinline__ uint64_t sdesc(uint32_t saddr, uint32_t lbo, uint32_t sbo, uint32_t layout) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4);
  d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32;
  d |= static_cast<uint64_t>(1u) << 46;
  d |= static_cast<uint64_t>(layout & 7u) << 61;
  return d;
}
constexpr uint32_t kLayoutSW128 = 2;

// kind::f16 instruction descriptor with B stored MN-major (N contiguous).
__host__ __device__ constexpr uint32_t idesc_bf16_f32_bmn(int M, int N) {
  return idesc_bf16_f32(M, N) | (1u << 16);
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
// Arrive on `bar` once every cp.async this thread issued so far has landed.
__device__ __forceinline__ void cp_async_arrive(uint32_t bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}
__device__ __forceinline__ float4 ld_shared_v4f(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(addr)
               : "memory");
  return v;
}
// Distributed shared memory: the address of the same offset in CTA `rank`.
__device__ __forceinline__ uint32_t map_peer(uint32_t saddr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
  return r;
}
// Arrive on an mbarrier of another CTA of the cluster, ordering this
// thread's earlier shared-memory accesses before the arrival.
__device__ __forceinline__ void mbar_arrive_remote(uint32_t raddr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(raddr) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait_cluster(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
// Whole-warp bounded wait on a barrier that threads of the other CTA arrive on.
__device__ __forceinline__ bool mbar_wait_warp_cluster(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                                       uint32_t* err) {
  uint64_t t0 = 0;
  for (uint32_t i = 0; i < kWaitLimitPolls; ++i) {
    const bool ok = mbar_try_wait_cluster(bar, parity);
    if (__all_sync(0xffffffffu, ok)) return true;
    if ((i & 63u) == 63u) {
      int stop = 0;
      if (lane_id() == 0) {
        const uint64_t now = global_timer_ns();
        if (t0 == 0) t0 = now;
        if (*abort_flag) stop = 1;
        else if (now - t0 > kWaitLimitNs) stop = 2;
      }
      stop = __shfl_sync(0xffffffffu, stop, 0);
      if (stop == 1) return false;
      if (stop == 2) break;
    }
  }
  if (lane_id() == 0) {
    *abort_flag = 1;
    raise_error(err, kErrTimeout);
  }
  __syncwarp();
  return false;
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t* v) {
  tmem_st16(taddr, v);
  tmem_st16(taddr + 16, v + 16);
}
__device__ __forceinline__ void tmem_st32f(uint32_t taddr, const float* v) {
  uint32_t u[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) u[i] = __float_as_uint(v[i]);
  tmem_st32(taddr, u);
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}


// Gather this CTA's NA atoms (64 latent columns each) of the tile's 64 rows.
// Lane l of each gather warp holds the global rows of tile rows l and l + 32.
template <int NA>
__device__ __forceinline__ void gather_tile(uint32_t dst0, const char* kv_b, int a0, int cur0, int cur1, int tid) {
#pragma unroll 4
  for (int i = 0; i < NA * 4; ++i) {
    const int x = i * 128 + tid;
    const int row = x / (NA * 8), cc = x % (NA * 8);
    const int v0 = __shfl_sync(0xffffffffu, cur0, row & 31);
    const int v1 = __shfl_sync(0xffffffffu, cur1, row & 31);
    const int s = row < 32 ? v0 : v1;
    const int kb = cc >> 3, c = cc & 7;
    const uint32_t dst = dst0 + kb * kAtomBytes + row * 128 + ((c ^ (row & 7)) << 4);
    const char* src = kv_b + (s >= 0 ? (static_cast<int64_t>(s) * kDqk + (a0 + kb) * 64) * 2 + c * 16 : 0);
    cp_async16(dst, src, s >= 0 ? 16u : 0u);
  }
}

// Single-thread bounded wait on a barrier that the other CTA arrives on.
__device__ __forceinline__ bool mbar_wait_cluster1(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                                   uint32_t* err) {
  const uint64_t t0 = global_timer_ns();
  for (uint32_t i = 0; i < kWaitLimitPolls; ++i) {
    if (mbar_try_wait_cluster(bar, parity)) return true;
    if ((i & 63u) == 63u) {
      if (*abort_flag) return false;
      if (global_timer_ns() - t0 > kWaitLimitNs) break;
    }
  }
  *abort_flag = 1;
  raise_error(err, kErrTimeout);
  return false;
}
// Bulk copy of `bytes` from this CTA's shared memory into the other CTA's,
// completing on the other CTA's barrier (addresses already mapped).
__device__ __forceinline__ void bulk_to_peer(uint32_t dst, uint32_t src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.shared::cta.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "r"(src), "r"(bytes), "r"(bar)
               : "memory");
}
// Pull the 128-byte line at p into L2 (a hint: no data returned, nothing to wait for).
__device__ __forceinline__ void prefetch_l2_line(const void* p) {
  asm volatile("prefetch.global.L2::evict_last [%0];" ::"l"(p));
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Wait until at most N of this thread's bulk groups still read their source.
template <int N>
__device__ __forceinline__ void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ void st_shared_f32(uint32_t addr, float v) {
  asm volatile("st.shared.f32 [%0], %1;" ::"r"(addr), "f"(v) : "memory");
}
__device__ __forceinline__ float ld_shared_f32(uint32_t addr) {
  float v;
  asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
  return v;
}
// Scale 32-column chunks [c0, c1) of this thread's O row in TMEM by f.
__device__ __forceinline__ void rescale_o_cols(uint32_t tl, int c0, int c1, float f) {
#pragma unroll 1
  for (int c = c0; c < c1; c += 32) {
    float o[32];
    tmem_ld32(tl + c, o);
#pragma unroll
    for (int i = 0; i < 32; ++i) o[i] *= f;
    tmem_st32f(tl + c, o);
  }
  tmem_st_wait();
}

__global__ void __launch_bounds__(kThreads, 1) attn_mla_tc_kernel(AttnParams P) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_addr(smem);
  const uint32_t bar0 = sbase + kOffBar;
  auto kv_full = [&](int i) { return bar0 + 8u * i; };
  auto kv_empty = [&](int i) { return bar0 + 8u * (kStages + i); };
  const uint32_t q_ready = bar0 + 8u * (2 * kStages + 0);
  const uint32_t s_full = bar0 + 8u * (2 * kStages + 1);
  const uint32_t s_empty = bar0 + 8u * (2 * kStages + 2);
  const uint32_t mma_done = bar0 + 8u * (2 * kStages + 3);
  const uint32_t fin = bar0 + 8u * (2 * kStages + 4);
  const uint32_t pside_done = bar0 + 8u * (2 * kStages + 5);  // P-side warps saw the last tile's statistics
  // double-buffered barriers, index [tile parity]
  enum {
    X_FULL,         // received partial logits landed (armed here, bulk copy from the other CTA)
    X_EMPTY,        // the other CTA has added our shipped partial (remote arrive)
    XOUT_WRITTEN,   // ship warps staged the outgoing partial
    XOUT_FREE,      // the outgoing bulk copy has read the staging buffer
    XIN_READ,       // softmax warps have added the received partial
    P_OWN_WRITTEN,  // softmax warps wrote their heads' P rows and statistics
    PEER_P_FREE,    // the other CTA's P buffer is free (its PV two tiles back is done; remote arrive)
    P_REMOTE_FULL,  // the other CTA's P rows and statistics landed (armed here, bulk copy)
    PV_READY,       // all P rows present and every O row rescaled: PV may run
    PV_DONE,        // PV of this buffer's last tile is done (tcgen05.commit)
    RED_FULL        // both softmax warps of each head published their tile max
  };
  auto dbar = [&](int which, int b) { return bar0 + 8u * (2 * kStages + 6 + 2 * which + b); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffMisc + 4);
  volatile int* gather_progress = reinterpret_cast<volatile int*>(smem + kOffMisc + 8);

  const int warp = threadIdx.x >> 5;
  const int lane = lane_id();
  const uint32_t crank = cluster_rank();  // 0: latent columns [0, 256), heads [0, 64); 1: [256, 576), [64, 128)
  const uint32_t peer = crank ^ 1u;
  const int a0 = crank == 0 ? 0 : kSplitCol / 64;  // first 64-column atom of this CTA
  const int natoms = crank == 0 ? kSplitCol / 64 : (kDqk - kSplitCol) / 64;
  // work item of the cluster
  const int item = blockIdx.x >> 1;
  const int sp = item % P.splits;
  const int r = item / P.splits;
  const int b = r / P.n_q;
  const int L = min(max(__ldg(P.ctx_len + b), 0), P.s_max);
  const int row0 = sp * P.rows_per_split;
  const int nrows = max(0, min(P.rows_per_split, P.k - row0));
  const int T = (nrows + kRows - 1) / kRows;
  const int32_t* sel = P.idx + static_cast<int64_t>(r) * P.k + row0;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(kv_full(i), 32 * kGatherWarps);
      mbar_init(kv_empty(i), 1);
    }
    mbar_init(q_ready, 32 * kSoftWarps);
    mbar_init(s_full, 1);
    mbar_init(s_empty, 192);  // 128 softmax threads + 64 ship threads read S
    mbar_init(mma_done, 1);
    mbar_init(fin, 128);
    mbar_init(pside_done, 64);
    for (int bb = 0; bb < 2; ++bb) {
      mbar_init(dbar(X_FULL, bb), 1);
      mbar_init(dbar(X_EMPTY, bb), 1);
      mbar_init(dbar(XOUT_WRITTEN, bb), 64);
      mbar_init(dbar(XOUT_FREE, bb), 1);
      mbar_init(dbar(XIN_READ, bb), 128);
      mbar_init(dbar(P_OWN_WRITTEN, bb), 128);
      mbar_init(dbar(PEER_P_FREE, bb), 1);
      mbar_init(dbar(P_REMOTE_FULL, bb), 1);
      mbar_init(dbar(PV_READY, bb), 192);  // 128 softmax threads + 64 P-side threads
      mbar_init(dbar(PV_DONE, bb), 1);
      mbar_init(dbar(RED_FULL, bb), 128);
      if (bb < T) {  // armed for tiles 0 and 1; later tiles re-arm one round ahead
        mbar_arrive_expect_tx(dbar(X_FULL, bb), kXBytes);
        mbar_arrive_expect_tx(dbar(P_REMOTE_FULL, bb), kPHalfBytes + kStatBytes);
      }
    }
    *abort_flag = 0;
    *gather_progress = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(smem_addr(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  cluster_sync_all();  // both CTAs' barriers exist (and are armed) before any remote arrival
  const uint32_t tmem = *tmem_slot;

  if (warp == kPrefetchWarp) {
    // ------------------------------------------- L2 prefetch of the rows --
    // Row reads from HBM take microseconds while a ring stage is held; pull
    // each tile's rows into L2 up to kPrefetchAhead tiles before its gather,
    // so the gather into the ring reads L2.  Lane l covers rows l and l + 32.
    const char* kv_b = reinterpret_cast<const char*>(P.kv) + static_cast<int64_t>(b) * P.s_max * kDqk * 2;
    const uint64_t t0 = global_timer_ns();
    for (int t = 1; t < T; ++t) {
      // stay at most kPrefetchAhead tiles ahead of the issued gathers (bounded)
      bool go = true;
      for (uint32_t i = 0; *gather_progress + kPrefetchAhead < t; ++i) {
        if ((i & 63u) == 63u && (*abort_flag || global_timer_ns() - t0 > kWaitLimitNs)) {
          go = false;
          break;
        }
        __nanosleep(200);
      }
      if (!__all_sync(0xffffffffu, go)) break;
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const int rr = t * kRows + hh * 32 + lane;
        const int s = rr < nrows ? __ldg(sel + rr) : -1;
        if (s >= 0 && s < L) {
          const char* row = kv_b + (static_cast<int64_t>(s) * kDqk + a0 * 64) * 2;
          for (int c = 0; c < natoms; ++c) prefetch_l2_line(row + c * 128);
        }
      }
    }
  } else if (warp < kGatherWarps) {
    // --------------------------------------------------- gather (cp.async) --
    const int tid = threadIdx.x;
    const char* kv_b = reinterpret_cast<const char*>(P.kv) + static_cast<int64_t>(b) * P.s_max * kDqk * 2;
    bool bad = false;
    int nx0 = (lane < nrows) ? __ldg(sel + lane) : -1;
    int nx1 = (lane + 32 < nrows) ? __ldg(sel + lane + 32) : -1;
    for (int j = 0; j < T; ++j) {
      const int st = j % kStages;
      int cur0 = nx0, cur1 = nx1;
      if (cur0 >= L) { bad = true; cur0 = -1; }
      if (cur1 >= L) { bad = true; cur1 = -1; }
      const int jn = (j + 1) * kRows + lane;
      nx0 = (j + 1 < T && jn < nrows) ? __ldg(sel + jn) : -1;
      nx1 = (j + 1 < T && jn + 32 < nrows) ? __ldg(sel + jn + 32) : -1;
      if (!mbar_wait_warp(kv_empty(st), ((j / kStages) & 1) ^ 1, abort_flag, P.err)) break;
      const uint32_t dst0 = sbase + kOffKV + st * kStageBytes;
      if (crank == 0) gather_tile<kSplitCol / 64>(dst0, kv_b, a0, cur0, cur1, tid);
      else gather_tile<(kDqk - kSplitCol) / 64>(dst0, kv_b, a0, cur0, cur1, tid);
      cp_async_arrive(kv_full(st));
      if (tid == 0) *gather_progress = j + 1;  // tiles whose gather has been issued
    }
    asm volatile("cp.async.wait_all;" ::: "memory");
    if (__any_sync(0xffffffffu, bad) && lane == 0) raise_error(P.err, kErrBadIndex);
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------- MMA issue --
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(kH, kRows);
      constexpr uint32_t idesc_o = idesc_bf16_f32_bmn(kH, kDvHalf);
      const uint64_t kv_desc0 = sdesc(sbase + kOffKV, 16, 1024, kLayoutSW128);      // K-major rows (logits)
      const uint64_t v_desc0 = sdesc(sbase + kOffKV, kAtomBytes, 1024, kLayoutSW128);  // MN-major columns (value)
      const uint64_t p_desc0 = sdesc(sbase + kOffP, 16, 1024, kLayoutSW128);
      const uint32_t q_t = tmem + kQCol, s_t = tmem + kSCol;
      bool ok = mbar_wait(q_ready, 0, abort_flag, P.err);
      int nq = 0, np = 0;
      uint64_t t0 = 0;
      uint32_t spins = 0;
      while (ok && np < T) {
        // O += P(np) V(np) once every P row is in place and O rows are rescaled
        if (np < nq && mbar_test_wait(dbar(PV_READY, np & 1), (np >> 1) & 1)) {
          tc_fence_after_sync();
          const uint64_t st_off = static_cast<uint64_t>(((np % kStages) * kStageBytes) >> 4);
          const uint64_t p_off = static_cast<uint64_t>(((np & 1) * kPBytes) >> 4);
#pragma unroll
          for (int kk = 0; kk < kRows / 16; ++kk)
            tc_mma_f16(tmem, p_desc0 + p_off + ((kk * 32) >> 4), v_desc0 + st_off + ((kk * 16 * 128) >> 4), idesc_o,
                       (np > 0 || kk > 0) ? 1u : 0u);
          tc_commit(kv_empty(np % kStages));
          tc_commit(dbar(PV_DONE, np & 1));
          ++np;
          spins = 0;
          continue;
        }
        // S(nq) = Q_c K_c(nq)^T once its rows landed and S(nq-1) was read
        if (nq < T && mbar_test_wait(kv_full(nq % kStages), (nq / kStages) & 1) &&
            mbar_test_wait(s_empty, (nq & 1) ^ 1)) {
          fence_proxy_async_smem();  // cp.async (generic proxy) writes -> tensor-core reads
          tc_fence_after_sync();
          const uint64_t kvs = kv_desc0 + static_cast<uint64_t>(((nq % kStages) * kStageBytes) >> 4);
          const int nk = natoms * 4;
          for (int kk = 0; kk < nk; ++kk) {
            const uint32_t b_off = (kk >> 2) * kAtomBytes + (kk & 3) * 32;
            tc_mma_f16_ts(s_t, q_t + kk * 8, kvs + (b_off >> 4), idesc_s, kk > 0 ? 1u : 0u);
          }
          tc_commit(s_full);
          ++nq;
          spins = 0;
          continue;
        }
        if ((++spins & 63u) == 0u) {
          const uint64_t now = global_timer_ns();
          if (t0 == 0 || spins == 64) t0 = now;
          if (*abort_flag) { ok = false; break; }
          if (now - t0 > kWaitLimitNs || spins > kWaitLimitPolls) {
            *abort_flag = 1;
            raise_error(P.err, kErrTimeout);
            ok = false;
          }
        }
      }
      tc_commit(mma_done);
      volatile int never = 0;
      mbar_wait(mma_done, 0, &never, P.err);
    }
    __syncwarp();
  } else {
    // ------------------------------------- Q to TMEM, then three roles --
    const int quarter = warp & 3;
    const int sub = (warp - (kGatherWarps + 1)) >> 2;  // which of the quarter's two warps
    const int h = quarter * 32 + lane;                 // head == TMEM lane
    const int hl = h & (kHHalf - 1);                   // index among its CTA's 64 heads
    const bool own = static_cast<uint32_t>(quarter >> 1) == crank;
    const uint32_t tl = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    {
      // this CTA's columns of q[r, h, :] as packed bf16 pairs (element 2i in
      // the low half of column i); the quarter's two warps take half each
      const uint4* qs = reinterpret_cast<const uint4*>(P.q + (static_cast<int64_t>(r) * kH + h) * kDqk + a0 * 64);
      for (int c = sub * natoms; c < (sub + 1) * natoms; ++c) {
        uint32_t u[16];
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          const uint4 x = __ldg(qs + c * 4 + v);
          u[4 * v + 0] = x.x;
          u[4 * v + 1] = x.y;
          u[4 * v + 2] = x.z;
          u[4 * v + 3] = x.w;
        }
        tmem_st16(tl + kQCol + c * 16, u);
      }
      tmem_st_wait();
      tc_fence_before_sync();
      mbar_arrive(q_ready);
    }
    const uint32_t p0 = sbase + kOffP;
    const uint32_t xin0 = sbase + kOffXin, xout0 = sbase + kOffXout;
    const uint32_t sto0 = sbase + kOffStOut, sti0 = sbase + kOffStIn;
    bool ok = true;
    float m_fin = -INFINITY, l_fin = 0.f;  // head h's final running max and sum
    int c_lo = 0, c_hi = 0;                // this thread's O columns in the epilogue

    if (own) {
      // ---------------------- softmax of this CTA's heads, 32 columns a warp --
      const int kh = sub;
      const bool leader = (hl == 0 && kh == 0);  // ships P rows; re-arms and releases the receive buffer
      float sreg[32], snext[32];
      float m_run = -INFINITY, l_half = 0.f;
      // validity of this lane's row in tiles [vbase, vbase + 32), loaded in
      // batches so that no global load is pending inside the loop (the
      // release-ordered remote arrivals below would wait for it)
      uint32_t vbits = 0;
      int vbase = -32;
      auto read_s = [&](float* dst) {
        tc_fence_after_sync();
        tmem_ld32(tl + kSCol + 32 * kh, dst);
        tc_fence_before_sync();
        mbar_arrive(s_empty);
      };
      // S(t) complete, tested without waiting; the whole warp agrees
      auto s_ready = [&](int t) { return __all_sync(0xffffffffu, mbar_test_wait(s_full, t & 1)); };
      bool have = false;  // sreg already holds S(j)
      for (int j = 0; ok && j < T; ++j) {
        const int bb = j & 1;
        const uint32_t ph = (j >> 1) & 1;
        if (j >= vbase + 32) {
          vbase = j;
          vbits = 0;
          for (int t = 0; t < 32 && j + t < T; ++t) {
            const int rr = (j + t) * kRows + kh * 32 + lane;
            const int ix = rr < nrows ? __ldg(sel + rr) : -1;
            vbits |= ((ix >= 0 && ix < L) ? 1u : 0u) << t;
          }
        }
        const uint32_t valid = __ballot_sync(0xffffffffu, ((vbits >> (j - vbase)) & 1u) != 0);
        if (!have) {
          if (!mbar_wait_warp(s_full, j & 1, abort_flag, P.err)) { ok = false; break; }
          read_s(sreg);
        }
        // the next tile's logits too if they are already there: its MMA then
        // runs under this tile's softmax (never wait for them here: they
        // hang on the next gather)
        have = j + 1 < T && s_ready(j + 1);
        if (have) read_s(snext);
        // S = S_0 + S_1: add the other CTA's partial for these heads
        if (!mbar_wait_warp_cluster(dbar(X_FULL, bb), ph, abort_flag, P.err)) { ok = false; break; }
        const uint32_t xb = xin0 + bb * kXBytes;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const float4 v = ld_shared_v4f(xb + ((kh * 8 + c) * kHHalf + hl) * 16);
          sreg[4 * c] += v.x;
          sreg[4 * c + 1] += v.y;
          sreg[4 * c + 2] += v.z;
          sreg[4 * c + 3] += v.w;
        }
        mbar_arrive(dbar(XIN_READ, bb));
        if (leader && mbar_wait(dbar(XIN_READ, bb), ph, abort_flag, P.err) && j + 2 < T) {
          mbar_arrive_expect_tx(dbar(X_FULL, bb), kXBytes);  // armed for tile j + 2 ...
          mbar_arrive_remote(map_peer(dbar(X_EMPTY, bb), peer));  // ... before the other CTA may send it
        }
        float mt = -INFINITY;
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const bool v = ((valid >> i) & 1u) != 0;
          sreg[i] = v ? sreg[i] * P.scale_log2 : -INFINITY;
          mt = fmaxf(mt, sreg[i]);
        }
        // tile max over all 64 columns: swap with the head's other warp
        const uint32_t red = sbase + kOffRed + bb * (2 * kHHalf * 4);
        st_shared_f32(red + (kh * kHHalf + hl) * 4, mt);
        mbar_arrive(dbar(RED_FULL, bb));
        if (!mbar_wait_warp(dbar(RED_FULL, bb), ph, abort_flag, P.err)) { ok = false; break; }
        mt = fmaxf(mt, ld_shared_f32(red + ((kh ^ 1) * kHHalf + hl) * 4));
        // move the running max only when the tile max exceeds it by > 8 (base 2)
        const bool move = mt > m_run + 8.f;
        const bool rescale_o = move && m_run != -INFINITY;
        if (__any_sync(0xffffffffu, rescale_o)) {
          // O must hold every previous tile before it is rescaled (PV of
          // tile j - 3 was awaited one tile ago, so this parity is unambiguous)
          if (j >= 1 && !mbar_wait_warp(dbar(PV_DONE, bb ^ 1), ((j - 1) >> 1) & 1, abort_flag, P.err)) {
            ok = false;
            break;
          }
          tc_fence_after_sync();
          rescale_o_cols(tl, kh * 128, kh * 128 + 128, rescale_o ? exp2f(m_run - mt) : 1.f);
        }
        if (move) {
          if (m_run != -INFINITY) l_half *= exp2f(m_run - mt);
          m_run = mt;
        }
        // P = 2^(s - m) in bf16, 128-byte-swizzled K-major; the buffer is free
        // once the PV two tiles back is done
        if (j >= 2 && !mbar_wait_warp(dbar(PV_DONE, bb), ((j - 2) >> 1) & 1, abort_flag, P.err)) {
          ok = false;
          break;
        }
        const uint32_t pb = p0 + bb * kPBytes;
        const uint32_t prow = pb + (h >> 3) * 1024 + (h & 7) * 128;
        float psum = 0.f;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          float p[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            p[e] = (m_run == -INFINITY) ? 0.f : fast_exp2(sreg[c * 8 + e] - m_run);
            psum += p[e];
          }
          st_shared_v4(prow + (((kh * 4 + c) ^ (h & 7)) << 4), pack_bf16(p[0], p[1]), pack_bf16(p[2], p[3]),
                       pack_bf16(p[4], p[5]), pack_bf16(p[6], p[7]));
        }
        l_half += psum;
        // statistics for the other CTA: running max, and each warp's partial sum
        const uint32_t so = sto0 + bb * kStatBytes;
        if (kh == 0) st_shared_f32(so + hl * 4, m_run);
        st_shared_f32(so + ((1 + kh) * kHHalf + hl) * 4, l_half);
        fence_proxy_async_smem();
        tc_fence_before_sync();
        mbar_arrive(dbar(P_OWN_WRITTEN, bb));
        mbar_arrive(dbar(PV_READY, bb));
        if (leader) {
          bool go = mbar_wait(dbar(P_OWN_WRITTEN, bb), ph, abort_flag, P.err);
          if (go && j >= 2) go = mbar_wait_cluster1(dbar(PEER_P_FREE, bb), ((j - 2) >> 1) & 1, abort_flag, P.err);
          if (go) {
            bulk_wait_read<0>();  // earlier copies have read P and the statistics
            const uint32_t pbar = map_peer(dbar(P_REMOTE_FULL, bb), peer);
            const uint32_t mine = pb + crank * kPHalfBytes;
            bulk_to_peer(map_peer(mine, peer), mine, kPHalfBytes, pbar);
            bulk_to_peer(map_peer(sti0 + bb * kStatBytes, peer), so, kStatBytes, pbar);
            bulk_commit();
          }
        }
        if (!have && j + 1 < T && s_ready(j + 1)) {
          read_s(snext);
          have = true;
        }
        if (have) {
#pragma unroll
          for (int i = 0; i < 32; ++i) sreg[i] = snext[i];
        }
      }
      if (leader) asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
      // both warps' partial sums of the last tile
      if (ok && T > 0) {
        mbar_arrive(fin);
        ok = mbar_wait_warp(fin, 0, abort_flag, P.err);
      }
      if (ok && T > 0) {
        const uint32_t so = sto0 + ((T - 1) & 1) * kStatBytes;
        m_fin = m_run;
        l_fin = ld_shared_f32(so + (kHHalf + hl) * 4) + ld_shared_f32(so + (2 * kHHalf + hl) * 4);
      }
      c_lo = kh * 128;
      c_hi = c_lo + 128;
    } else if (sub == 0) {
      // ------------ ship: partial logits of the other CTA's heads, per tile --
      const bool leader = (hl == 0);
      for (int j = 0; ok && j < T; ++j) {
        const int bb = j & 1;
        const uint32_t ph = (j >> 1) & 1;
        if (!mbar_wait_warp(s_full, j & 1, abort_flag, P.err)) { ok = false; break; }
        tc_fence_after_sync();
        float s[kRows];
        tmem_ld32(tl + kSCol, s);
        tmem_ld32(tl + kSCol + 32, s + 32);
        tc_fence_before_sync();
        mbar_arrive(s_empty);
        if (j >= 2 && !mbar_wait_warp(dbar(XOUT_FREE, bb), ((j - 2) >> 1) & 1, abort_flag, P.err)) {
          ok = false;
          break;
        }
        const uint32_t xo = xout0 + bb * kXBytes;
#pragma unroll
        for (int c = 0; c < kRows / 4; ++c)
          asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(xo + (c * kHHalf + hl) * 16), "f"(s[4 * c]),
                       "f"(s[4 * c + 1]), "f"(s[4 * c + 2]), "f"(s[4 * c + 3])
                       : "memory");
        fence_proxy_async_smem();
        mbar_arrive(dbar(XOUT_WRITTEN, bb));
        if (leader) {
          bool go = mbar_wait(dbar(XOUT_WRITTEN, bb), ph, abort_flag, P.err);
          if (go && j >= 2) go = mbar_wait_cluster1(dbar(X_EMPTY, bb), ((j - 2) >> 1) & 1, abort_flag, P.err);
          if (go) {
            bulk_to_peer(map_peer(xin0 + bb * kXBytes, peer), xo, kXBytes, map_peer(dbar(X_FULL, bb), peer));
            bulk_commit();
            if (j >= 1) {
              bulk_wait_read<1>();  // the copy of tile j - 1 has read its staging buffer
              mbar_arrive(dbar(XOUT_FREE, bb ^ 1));
            }
          }
        }
      }
      if (leader) asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
      // the other CTA's statistics of these heads after the last tile, once
      // the P-side warps (which waited on every tile's copy) have seen them
      if (ok && T > 0) ok = mbar_wait_warp(pside_done, 0, abort_flag, P.err);
      if (ok && T > 0) {
        const uint32_t si = sti0 + ((T - 1) & 1) * kStatBytes;
        m_fin = ld_shared_f32(si + hl * 4);
        l_fin = ld_shared_f32(si + (kHHalf + hl) * 4) + ld_shared_f32(si + (2 * kHHalf + hl) * 4);
      }
      c_lo = 128;
      c_hi = 256;
    } else {
      // -------- P side: the other CTA's P rows and statistics, O rescaling --
      const bool leader = (hl == 0);
      float m_prev = -INFINITY;
      for (int j = 0; ok && j < T; ++j) {
        const int bb = j & 1;
        const uint32_t ph = (j >> 1) & 1;
        if (leader && j >= 2 && mbar_wait(dbar(PV_DONE, bb), ((j - 2) >> 1) & 1, abort_flag, P.err)) {
          // P buffer bb is free again: arm it for tile j, then let the other CTA fill it
          mbar_arrive_expect_tx(dbar(P_REMOTE_FULL, bb), kPHalfBytes + kStatBytes);
          mbar_arrive_remote(map_peer(dbar(PEER_P_FREE, bb), peer));
        }
        if (!mbar_wait_warp_cluster(dbar(P_REMOTE_FULL, bb), ph, abort_flag, P.err)) { ok = false; break; }
        const float m_new = ld_shared_f32(sti0 + bb * kStatBytes + hl * 4);
        const bool rescale_o = m_new != m_prev && m_prev != -INFINITY;
        if (__any_sync(0xffffffffu, rescale_o)) {
          // (P_REMOTE_FULL of tile j implies PV of tile j - 2 is done)
          if (j >= 1 && !mbar_wait_warp(dbar(PV_DONE, bb ^ 1), ((j - 1) >> 1) & 1, abort_flag, P.err)) {
            ok = false;
            break;
          }
          tc_fence_after_sync();
          rescale_o_cols(tl, 0, kDvHalf, rescale_o ? exp2f(m_prev - m_new) : 1.f);
        }
        m_prev = m_new;
        tc_fence_before_sync();
        mbar_arrive(dbar(PV_READY, bb));
      }
      if (ok && T > 0) mbar_arrive(pside_done);
      if (ok && T > 0) {
        const uint32_t si = sti0 + ((T - 1) & 1) * kStatBytes;
        m_fin = m_prev;
        l_fin = ld_shared_f32(si + (kHHalf + hl) * 4) + ld_shared_f32(si + (2 * kHHalf + hl) * 4);
      }
      c_lo = 0;
      c_hi = 128;
    }
    // ------------------------------------------------------------ output --
    // every role has seen PV of tile T - 3 complete (directly, or through the
    // other CTA's P rows of tile T - 1), so this parity is unambiguous
    if (ok && T >= 1) ok = mbar_wait_warp(dbar(PV_DONE, (T - 1) & 1), ((T - 1) >> 1) & 1, abort_flag, P.err);
    if (ok) {
      tc_fence_after_sync();
      const int64_t rh = static_cast<int64_t>(r) * kH + h;
      const bool stats_writer = own ? (sub == 0) : (sub == 1);  // one thread per head
      if (P.splits == 1) {
        const float inv = l_fin > 0.f ? 1.f / l_fin : 0.f;
        __nv_bfloat16* dst = P.out + rh * kDv + crank * kDvHalf;
#pragma unroll 1
        for (int c = c_lo; c < c_hi; c += 32) {
          float o[32];
          if (T >= 1) tmem_ld32(tl + c, o);
          else
            for (int i = 0; i < 32; ++i) o[i] = 0.f;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint4 v;
            v.x = pack_bf16(o[q * 8 + 0] * inv, o[q * 8 + 1] * inv);
            v.y = pack_bf16(o[q * 8 + 2] * inv, o[q * 8 + 3] * inv);
            v.z = pack_bf16(o[q * 8 + 4] * inv, o[q * 8 + 5] * inv);
            v.w = pack_bf16(o[q * 8 + 6] * inv, o[q * 8 + 7] * inv);
            *reinterpret_cast<uint4*>(dst + c + q * 8) = v;
          }
        }
        if (P.lse != nullptr && crank == 0 && stats_writer)
          P.lse[rh] = l_fin > 0.f ? (m_fin + log2f(l_fin)) * 0.6931471805599453f : -INFINITY;
      } else {
        const int64_t it = (static_cast<int64_t>(r) * P.splits + sp) * 2 + crank;
        float* dst = P.part_o + (it * kH + h) * kDvHalf;
#pragma unroll 1
        for (int c = c_lo; c < c_hi; c += 32) {
          float o[32];
          if (T >= 1) tmem_ld32(tl + c, o);
          else
            for (int i = 0; i < 32; ++i) o[i] = 0.f;
#pragma unroll
          for (int q = 0; q < 8; ++q)
            *reinterpret_cast<float4*>(dst + c + q * 4) = make_float4(o[q * 4], o[q * 4 + 1], o[q * 4 + 2], o[q * 4 + 3]);
        }
        if (own && stats_writer) {
          const int64_t ms = static_cast<int64_t>(r) * P.splits + sp;
          P.part_ml[(ms * 2 + 0) * kH + h] = m_fin;
          P.part_ml[(ms * 2 + 1) * kH + h] = l_fin;
        }
      }
    }
  }

  tc_fence_before_sync();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after_sync();
    tmem_dealloc(tmem, kTmemCols);
  }
  cluster_sync_all();  // no CTA leaves while the other may still touch its shared memory
}
}  // namespace
}  // namespace dsa

namespace dsa {
namespace {

constexpr int kMaxSplits = 16;
constexpr int kCombineHeads = 8;  // heads per combine block

// Merge the per-split partial outputs of each query: O = sum_i 2^(m_i - M) O_i
// / sum_i 2^(m_i - M) l_i with M = max_i m_i (base-2 log-sum-exp combine).
// Block = (query, group of 8 heads); 256 threads, 4 output columns a step.
__global__ void __launch_bounds__(256) attn_combine_kernel(const float* __restrict__ part_o,
                                                           const float* __restrict__ part_ml, int splits,
                                                           __nv_bfloat16* __restrict__ out, float* __restrict__ lse) {
  __shared__ float coef[kMaxSplits][kCombineHeads];
  const int r = blockIdx.x;
  const int h0 = blockIdx.y * kCombineHeads;
  const int tid = threadIdx.x;
  if (tid < kCombineHeads) {
    const int h = h0 + tid;
    float M = -INFINITY;
    for (int i = 0; i < splits; ++i) {
      const int64_t it = static_cast<int64_t>(r) * splits + i;
      const float m = part_ml[(it * 2 + 0) * kH + h];
      const float l = part_ml[(it * 2 + 1) * kH + h];
      if (l > 0.f) M = fmaxf(M, m);
    }
    float Ls = 0.f;
    for (int i = 0; i < splits; ++i) {
      const int64_t it = static_cast<int64_t>(r) * splits + i;
      const float m = part_ml[(it * 2 + 0) * kH + h];
      const float l = part_ml[(it * 2 + 1) * kH + h];
      const float wgt = (l > 0.f) ? exp2f(m - M) : 0.f;
      coef[i][tid] = wgt;
      Ls += wgt * l;
    }
    const float inv = Ls > 0.f ? 1.f / Ls : 0.f;
    for (int i = 0; i < splits; ++i) coef[i][tid] *= inv;
    if (lse != nullptr)
      lse[static_cast<int64_t>(r) * kH + h] = Ls > 0.f ? (M + log2f(Ls)) * 0.6931471805599453f : -INFINITY;
  }
  __syncthreads();
#pragma unroll
  for (int itr = 0; itr < kCombineHeads * (kDv / 4) / 256; ++itr) {
    const int x = itr * 256 + tid;
    const int hl = x / (kDv / 4);
    const int c4 = x % (kDv / 4);
    const int h = h0 + hl;
    const int hv = c4 / (kDvHalf / 4);
    const int cc = (c4 % (kDvHalf / 4)) * 4;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int i = 0; i < splits; ++i) {
      const int64_t it = (static_cast<int64_t>(r) * splits + i) * 2 + hv;
      const float4 o = __ldg(reinterpret_cast<const float4*>(part_o + (it * kH + h) * kDvHalf + cc));
      const float c = coef[i][hl];
      acc.x = fmaf(c, o.x, acc.x);
      acc.y = fmaf(c, o.y, acc.y);
      acc.z = fmaf(c, o.z, acc.z);
      acc.w = fmaf(c, o.w, acc.w);
    }
    uint2 v;
    v.x = pack_bf16(acc.x, acc.y);
    v.y = pack_bf16(acc.z, acc.w);
    *reinterpret_cast<uint2*>(out + (static_cast<int64_t>(r) * kH + h) * kDv + c4 * 4) = v;
  }
}

struct SplitPlan {
  int splits, rows_per_split;
};

// Splits of each query's selected list so that clusters (2 SMs each) cover
// the GPU: none when the queries alone fill it.
SplitPlan plan_splits(int64_t R, int k, int num_sms) {
  SplitPlan p;
  int s = 1;
  if (R * 2 < num_sms) s = static_cast<int>(std::max<int64_t>(1, num_sms / (R * 2)));
  s = std::min(s, kMaxSplits);
  int rps = (k + s - 1) / s;
  rps = (rps + kRows - 1) / kRows * kRows;
  p.rows_per_split = std::max(rps, kRows);
  p.splits = (k + p.rows_per_split - 1) / p.rows_per_split;
  return p;
}

size_t scratch_bytes(int64_t R, const SplitPlan& p) {
  if (p.splits <= 1) return 0;
  const size_t items = static_cast<size_t>(R) * p.splits * 2;
  return items * kH * kDvHalf * 4 + items * 2 * kH * 4;
}

}  // namespace

bool attn_tc_supported(int H, int d_qk, int d_v, int KVH) {
  return H == kH && d_qk == kDqk && d_v == kDv && KVH == 1;
}

size_t attn_workspace_bytes(int B, int n_q, int H, int d_qk, int d_v, int KVH, int k, int dtype) {
  if (dtype != DSA_BF16 || !attn_tc_supported(H, d_qk, d_v, KVH)) return 0;
  const int64_t R = static_cast<int64_t>(B) * n_q;
  // the split plan depends on the SM count; size for the largest plan any
  // B200-class part (<= 256 SMs) would pick
  return scratch_bytes(R, plan_splits(R, k, 256));
}

size_t attn_scratch_bytes(int B, int n_q, int k, int num_sms) {
  const int64_t R = static_cast<int64_t>(B) * n_q;
  if (R == 0) return 0;
  return scratch_bytes(R, plan_splits(R, k, num_sms));
}

dsa_status_t attn_tc(const AttnArgs& a) {
  const int64_t R = static_cast<int64_t>(a.B) * a.n_q;
  if (R == 0) return DSA_OK;
  const int num_sms = device_sm_count(a.device);
  const SplitPlan p = plan_splits(R, a.k, num_sms);
  if (R * p.splits * 2 > INT32_MAX) return DSA_ERR_UNSUPPORTED;
  AttnParams P;
  P.q = static_cast<const uint16_t*>(a.q);
  P.kv = static_cast<const uint16_t*>(a.kv);
  P.idx = a.idx;
  P.ctx_len = a.ctx_len;
  P.out = static_cast<__nv_bfloat16*>(a.out);
  P.lse = a.lse;
  P.n_q = a.n_q;
  P.s_max = a.s_max;
  P.k = a.k;
  P.splits = p.splits;
  P.rows_per_split = p.rows_per_split;
  P.scale_log2 = a.sm_scale * 1.4426950408889634f;
  P.err = a.err;
  P.part_o = nullptr;
  P.part_ml = nullptr;
  if (p.splits > 1) {
    const size_t need = scratch_bytes(R, p);
    if (a.ws == nullptr || a.ws_bytes < need) return DSA_ERR_WORKSPACE;
    const size_t items = static_cast<size_t>(R) * p.splits * 2;
    P.part_o = static_cast<float*>(a.ws);
    P.part_ml = P.part_o + items * kH * kDvHalf;
  }
  static bool attr_done[64] = {};
  if (a.device < 64 && !attr_done[a.device]) {
    if (cudaFuncSetAttribute(attn_mla_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes) !=
        cudaSuccess)
      return DSA_ERR_CUDA;
    attr_done[a.device] = true;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(R * p.splits * 2), 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = a.stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, attn_mla_tc_kernel, P) != cudaSuccess) return DSA_ERR_CUDA;
  if (p.splits > 1) {
    attn_combine_kernel<<<dim3(static_cast<unsigned>(R), kH / kCombineHeads), 256, 0, a.stream>>>(
        P.part_o, P.part_ml, p.splits, P.out, a.lse);
    if (cudaGetLastError() != cudaSuccess) return DSA_ERR_CUDA;
  }
  return DSA_OK;
}

}  // namespace dsa
