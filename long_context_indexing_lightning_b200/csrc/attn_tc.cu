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
// list).  CTA c owns latent columns [256c, 256c + 256) and rope columns
// [512 + 32c, 544 + 32c).  Per 64-row tile, each CTA
//   * gathers only its own columns of the selected rows (cp.async, 16 bytes a
//     thread, into a 3-stage ring in the swizzled K-major layouts the MMA
//     reads: 128-byte swizzle for the latent part, 64-byte for the rope part;
//     padding and out-of-range rows are zero filled), helped by a warp that
//     pulls the rows of the next tiles into L2 ahead of time,
//   * computes its partial logits S_c = Q_c K_c^T for all 128 heads (M = 128,
//     N = 64, Q_c held in tensor memory),
//   * swaps partials with the other CTA (32 KB, one bulk copy into the other
//     CTA's shared memory), so both hold the same S = S_0 + S_1 (fp32
//     addition is commutative: the two sums are bit-identical) and run the
//     same online softmax over all heads (base 2; the running max only moves,
//     and O is rescaled in TMEM, when a tile max exceeds it by more than 8),
//   * accumulates its 256-column half of the output, O_c += P V_c, in TMEM
//     (V_0 = latent columns [0, 256), V_1 = [256, 512): each CTA's value half
//     lies inside the columns it already gathered).
// The swap of tile j+1 is issued before the softmax of tile j and lands in
// the second of two receive buffers, so the copy overlaps the softmax; one
// warp does the copies and the cross-CTA signals.
// Warps: 0-3 gather, 4 issues tcgen05.mma, 5-12 softmax (two per TMEM lane
// quarter, thread = head = TMEM lane, 32 of the tile's 64 columns each), 13
// L2 prefetch, 14 copies.  Long selections are split across clusters and
// merged by a small combine kernel (log-sum-exp weights).  Every wait is
// bounded.
#include "dsa_common.cuh"
#include "dsa_internal.h"

namespace dsa {
namespace {

constexpr int kH = 128;                  // heads == MMA M
constexpr int kDqk = 576;                // latent 512 + rope 64
constexpr int kDv = 512;
constexpr int kDvHalf = 256;
constexpr int kRows = 64;                // selected rows per tile (MMA N of S, K of PV)
constexpr int kLatCols = 256;            // latent columns per CTA (also its value half)
constexpr int kLatAtoms = kLatCols / 64; // 64-column, 128-byte-swizzled atoms per tile
constexpr int kRopeCols = 32;            // rope columns per CTA
constexpr int kAtomBytes = kRows * 128;  // one latent atom of one tile: 8 KB
constexpr int kRopeBytes = kRows * 64;   // the rope piece of one tile (64-byte swizzle): 4 KB
constexpr int kStageBytes = kLatAtoms * kAtomBytes + kRopeBytes;  // 36 KB
constexpr int kQk = kLatCols + kRopeCols;  // 288 logit columns per CTA: 18 MMA K-steps
constexpr int kStages = 3;
constexpr int kPrefetchAhead = 6;        // tiles whose rows are pulled into L2 ahead of their gather
constexpr int kGatherWarps = 4;
constexpr int kMmaWarp = 4;
constexpr int kSoftWarps = 8;
constexpr int kSoftThreads = 32 * kSoftWarps;
constexpr int kPrefetchWarp = kGatherWarps + 1 + kSoftWarps;  // 13
constexpr int kCommWarp = kPrefetchWarp + 1;                   // 14
constexpr int kThreads = 32 * (kCommWarp + 1);                 // 480
// tensor memory: O half [0, 256), Q columns [256, 400), S [400, 464), P [464, 496)
// (P as bf16 pairs: the A operand of the value MMA)
constexpr int kTmemCols = 512;
constexpr int kQCol = 256;
constexpr int kSCol = kQCol + kQk / 2;
constexpr int kPCol = kSCol + kRows;
static_assert(kPCol + kRows / 2 <= kTmemCols, "tensor memory");

// shared memory map (from a 1024-aligned base)
constexpr int kXBytes = kH * kRows * 4;  // partial logits: [16 x 4 rows][128 heads] fp32
constexpr int kOffKV = 0;
constexpr int kOffXin = kOffKV + kStages * kStageBytes;  // the other CTA's partials, [tile parity]
constexpr int kOffXout = kOffXin + 2 * kXBytes;  // this CTA's partial, for the bulk copy
constexpr int kOffRed = kOffXout + kXBytes;  // tile max of each softmax warp: [2][2 warps][128]
// barriers: kv_full[3], kv_empty[3], then the 17 named in the kernel
constexpr int kNumBars = 2 * kStages + 17;
constexpr int kOffBar = kOffRed + 2 * 2 * kH * 4;
constexpr int kOffMisc = kOffBar + kNumBars * 8;
constexpr int kSmemBytes = kOffMisc + 16 + 1024;
static_assert(kSmemBytes <= 232448, "shared memory");
static_assert(kStageBytes % 1024 == 0, "ring stages must stay 1024-aligned");
// output staging: one slot per softmax warp in the ring, 32 rows of 144 bytes
constexpr int kOutSlotBytes = 32 * 144;
static_assert(kSoftWarps * kOutSlotBytes <= kStages * kStageBytes, "output staging fits in the ring");

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
// Gather warp w covers tile rows [16w, 16w + 16); in group g its lane l moves
// 16-byte chunk l % 8 of every atom of row 16w + 4g + l / 8, whose cache row
// is rows[g] (-1: zero fill).  No per-copy shuffles or divisions.
template <int NA>
__device__ __forceinline__ void gather_tile(uint32_t dst0, const char* kv_b, int a0, const int* rows, int w, int lane) {
  const int c = lane & 7;
#pragma unroll
  for (int g = 0; g < 4; ++g) {
    const int row = w * 16 + g * 4 + (lane >> 3);
    const int s = rows[g];
    const char* src = kv_b + (s >= 0 ? (static_cast<int64_t>(s) * kDqk + a0 * 64) * 2 + c * 16 : 0);
    const uint32_t dst = dst0 + row * 128 + ((c ^ (row & 7)) << 4);
    const uint32_t nbytes = s >= 0 ? 16u : 0u;
    const int step = s >= 0 ? 128 : 0;
#pragma unroll
    for (int a = 0; a < NA; ++a) cp_async16(dst + a * kAtomBytes, src + a * step, nbytes);
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
__device__ __forceinline__ void st_shared_u4(uint32_t addr, uint4 v) {
  asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}
__device__ __forceinline__ uint4 ld_shared_u4(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr)
               : "memory");
  return v;
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

// Gather this CTA's 32 rope columns of the tile's 64 rows into the piece at
// dst0: 64-byte rows, 64-byte swizzle (16-byte chunk c of row r sits at chunk
// c ^ ((r & 7) >> 1)).  Gather warp w covers rows [16w, 16w + 16); in group g
// its lane l moves chunk l % 4 of row 16w + 8g + l / 4, whose cache row is
// rows[g] (-1: zero fill).
__device__ __forceinline__ void gather_rope(uint32_t dst0, const char* kv_b, int col0, const int* rows, int w,
                                            int lane) {
  const int c = lane & 3;
#pragma unroll
  for (int g = 0; g < 2; ++g) {
    const int row = w * 16 + g * 8 + (lane >> 2);
    const int s = rows[g];
    const char* src = kv_b + (s >= 0 ? (static_cast<int64_t>(s) * kDqk + col0) * 2 + c * 16 : 0);
    const uint32_t dst = dst0 + (row >> 3) * 512 + (row & 7) * 64 + ((c ^ ((row & 7) >> 1)) << 4);
    cp_async16(dst, src, s >= 0 ? 16u : 0u);
  }
}
constexpr uint32_t kLayoutSW64 = 4;

__global__ void __launch_bounds__(kThreads, 1) attn_mla_tc_kernel(AttnParams P) {
  // (the set-up below reads no global memory: it runs before the wait for
  // the previous kernel, under its tail)
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_addr(smem);
  const uint32_t bar0 = sbase + kOffBar;
  auto kv_full = [&](int i) { return bar0 + 8u * i; };
  auto kv_empty = [&](int i) { return bar0 + 8u * (kStages + i); };
  const uint32_t nb0 = bar0 + 8u * (2 * kStages);
  const uint32_t q_ready = nb0 + 0;
  const uint32_t s_full = nb0 + 8;        // S(j) in TMEM (tcgen05.commit)
  const uint32_t s_empty = nb0 + 16;      // every softmax thread has read S(j)
  const uint32_t mma_done = nb0 + 24;
  const uint32_t fin = nb0 + 32;          // final partial sums published
  const uint32_t xout_written = nb0 + 40; // every softmax thread has written its partial of tile j
  const uint32_t xout_free = nb0 + 48;    // the bulk copy of tile j has read xout
  const uint32_t pv_ready = nb0 + 56;     // P of tile j written and O rescaled: PV may run
  const uint32_t pv_done = nb0 + 64;      // PV of tile j done (tcgen05.commit)
  // [tile parity]:
  auto red_full = [&](int bb) { return nb0 + 72 + 8u * bb; };   // tile max published
  auto x_full = [&](int bb) { return nb0 + 88 + 8u * bb; };     // the other CTA's partial landed in xin[bb] (tx)
  auto x_empty = [&](int bb) { return nb0 + 104 + 8u * bb; };   // the other CTA has added what we sent to its xin[bb]
  auto xin_read = [&](int bb) { return nb0 + 120 + 8u * bb; };  // every softmax thread has added xin[bb]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffMisc + 4);
  volatile int* gather_progress = reinterpret_cast<volatile int*>(smem + kOffMisc + 8);

  const int warp = threadIdx.x >> 5;
  const int lane = lane_id();
  const uint32_t crank = cluster_rank();  // latent columns [256c, 256c + 256), rope [512 + 32c, 544 + 32c)
  const uint32_t peer = crank ^ 1u;
  const int a0 = crank * kLatAtoms;                       // first 64-column latent atom of this CTA
  const int rope0 = kLatCols * 2 + crank * kRopeCols;     // first rope column of this CTA
  // work item of the cluster
  const int item = blockIdx.x >> 1;
  const int sp = item % P.splits;
  const int r = item / P.splits;
  const int b = r / P.n_q;
  const int row0 = sp * P.rows_per_split;
  const int nrows = max(0, min(P.rows_per_split, P.k - row0));
  const int T = (nrows + kRows - 1) / kRows;
  const int32_t* sel = P.idx + static_cast<int64_t>(r) * P.k + row0;
  const char* kv_b = reinterpret_cast<const char*>(P.kv) + static_cast<int64_t>(b) * P.s_max * kDqk * 2;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(kv_full(i), 32 * kGatherWarps);
      mbar_init(kv_empty(i), 1);
    }
    mbar_init(q_ready, kSoftThreads);
    mbar_init(s_full, 1);
    mbar_init(s_empty, kSoftThreads);
    mbar_init(mma_done, 1);
    mbar_init(fin, kSoftThreads);
    for (int bb = 0; bb < 2; ++bb) {
      mbar_init(x_full(bb), 1);
      mbar_init(x_empty(bb), 1);
      mbar_init(xin_read(bb), kSoftThreads);
      if (bb < T) mbar_arrive_expect_tx(x_full(bb), kXBytes);  // armed for tiles 0, 1; later re-armed ahead
    }
    mbar_init(xout_written, kSoftThreads);
    mbar_init(xout_free, 1);
    mbar_init(pv_ready, kSoftThreads);
    mbar_init(pv_done, 1);
    mbar_init(red_full(0), kSoftThreads);
    mbar_init(red_full(1), kSoftThreads);
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
  pdl_wait();
  const int L = min(max(__ldg(P.ctx_len + b), 0), P.s_max);

  if (warp == kCommWarp) {
    // --------------------------------------- copies and cross-CTA signals --
    // Lane 0 issues the bulk copies; lane 1, which has none in flight, sends
    // the remote signals (a release-ordered arrive from a thread with a copy
    // in flight waits for that copy).
    if (lane == 0) {
      for (int j = 0; j < T; ++j) {
        const int bb = j & 1;
        // this CTA's partial of tile j, once written and once the other CTA
        // has added the one that last used its buffer (tile j - 2)
        if (!mbar_wait(xout_written, j & 1, abort_flag, P.err)) break;
        if (j >= 2 && !mbar_wait_cluster1(x_empty(bb), ((j - 2) >> 1) & 1, abort_flag, P.err)) break;
        bulk_to_peer(map_peer(sbase + kOffXin + bb * kXBytes, peer), sbase + kOffXout, kXBytes,
                     map_peer(x_full(bb), peer));
        bulk_commit();
        bulk_wait_read<0>();
        mbar_arrive(xout_free);
      }
      asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
    } else if (lane == 1) {
      // our receive buffer [j & 1] is free once tile j's partial was added here
      for (int j = 0; j + 2 < T; ++j) {
        if (!mbar_wait(xin_read(j & 1), (j >> 1) & 1, abort_flag, P.err)) break;
        mbar_arrive_remote(map_peer(x_empty(j & 1), peer));
      }
    }
    __syncwarp();
  } else if (warp == kPrefetchWarp) {
    // ------------------------------------------- L2 prefetch of the rows --
    // Row reads from HBM take microseconds while a ring stage is held; pull
    // each tile's rows into L2 up to kPrefetchAhead tiles before its gather,
    // so the gather into the ring reads L2.  Lane l covers rows l and l + 32.
    // The ring's first kStages tiles are gathered at once; prefetching starts
    // behind those gathers (issued ahead of them, the prefetches of a whole
    // GPU delay the first tiles by microseconds).
    const uint64_t t0 = global_timer_ns();
    const int first = min(T, kStages);
    for (int t = kStages; t < T; ++t) {
      // stay at most kPrefetchAhead tiles ahead of the issued gathers (bounded)
      bool go = true;
      for (uint32_t i = 0; *gather_progress < first || *gather_progress + kPrefetchAhead < t; ++i) {
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
          const char* row = kv_b + static_cast<int64_t>(s) * kDqk * 2;
          for (int c = 0; c < kLatAtoms; ++c) prefetch_l2_line(row + (a0 + c) * 128);
          prefetch_l2_line(row + kLatCols * 4);  // the line holding both CTAs' rope columns
        }
      }
    }
  } else if (warp < kGatherWarps) {
    // --------------------------------------------------- gather (cp.async) --
    bool bad = false;
    const int myrow = warp * 16 + (lane >> 3);  // + 4 g: this lane's rows of each tile
    const int myrope = warp * 16 + (lane >> 2);  // + 8 g: this lane's rope rows
    int nx[4], rnx[2];
#pragma unroll
    for (int g = 0; g < 4; ++g) nx[g] = (myrow + 4 * g < nrows) ? __ldg(sel + myrow + 4 * g) : -1;
#pragma unroll
    for (int g = 0; g < 2; ++g) rnx[g] = (myrope + 8 * g < nrows) ? __ldg(sel + myrope + 8 * g) : -1;
    for (int j = 0; j < T; ++j) {
      const int st = j % kStages;
      int cur[4], rcur[2];
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        cur[g] = nx[g];
        if (cur[g] >= L) { bad = true; cur[g] = -1; }
        const int rn = (j + 1) * kRows + myrow + 4 * g;
        nx[g] = (j + 1 < T && rn < nrows) ? __ldg(sel + rn) : -1;
      }
#pragma unroll
      for (int g = 0; g < 2; ++g) {
        rcur[g] = rnx[g] < L ? rnx[g] : -1;  // (out-of-range rows are flagged above)
        const int rn = (j + 1) * kRows + myrope + 8 * g;
        rnx[g] = (j + 1 < T && rn < nrows) ? __ldg(sel + rn) : -1;
      }
      if (!mbar_wait_warp(kv_empty(st), ((j / kStages) & 1) ^ 1, abort_flag, P.err)) break;
      const uint32_t dst0 = sbase + kOffKV + st * kStageBytes;
      gather_tile<kLatAtoms>(dst0, kv_b, a0, cur, warp, lane);
      gather_rope(dst0 + kLatAtoms * kAtomBytes, kv_b, rope0, rcur, warp, lane);
      cp_async_arrive(kv_full(st));
      if (threadIdx.x == 0) *gather_progress = j + 1;  // tiles whose gather has been issued
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
      const uint64_t rope_desc0 = sdesc(sbase + kOffKV + kLatAtoms * kAtomBytes, 16, 512, kLayoutSW64);  // K-major rope rows
      const uint32_t q_t = tmem + kQCol, s_t = tmem + kSCol, p_t = tmem + kPCol;
      bool ok = mbar_wait(q_ready, 0, abort_flag, P.err);
      int nq = 0, np = 0;
      uint64_t t0 = 0;
      uint32_t spins = 0;
      while (ok && np < T) {
        // O += P(np) V(np) once P is written and O rescaled (frees the tile's stage)
        if (np < nq && mbar_test_wait(pv_ready, np & 1)) {
          tc_fence_after_sync();
          const uint64_t st_off = static_cast<uint64_t>(((np % kStages) * kStageBytes) >> 4);
#pragma unroll
          for (int kk = 0; kk < kRows / 16; ++kk)
            tc_mma_f16_ts(tmem, p_t + kk * 8, v_desc0 + st_off + ((kk * 16 * 128) >> 4), idesc_o,
                          (np > 0 || kk > 0) ? 1u : 0u);
          tc_commit(kv_empty(np % kStages));
          tc_commit(pv_done);
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
#pragma unroll
          for (int kk = 0; kk < kLatAtoms * 4; ++kk) {
            const uint32_t b_off = (kk >> 2) * kAtomBytes + (kk & 3) * 32;
            tc_mma_f16_ts(s_t, q_t + kk * 8, kvs + (b_off >> 4), idesc_s, kk > 0 ? 1u : 0u);
          }
          const uint64_t ropes = rope_desc0 + static_cast<uint64_t>(((nq % kStages) * kStageBytes) >> 4);
#pragma unroll
          for (int kk = 0; kk < kRopeCols / 16; ++kk)
            tc_mma_f16_ts(s_t, q_t + (kLatAtoms * 4 + kk) * 8, ropes + ((kk * 32) >> 4), idesc_s, 1u);
          tc_commit(s_full);
          ++nq;
          spins = 0;
          continue;
        }
        // nothing to issue: back off so this lane does not take issue slots
        // and shared-memory bandwidth from the gather and softmax warps
        __nanosleep(32);
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
    // ------------------------------------------- softmax (all 128 heads) --
    const int quarter = warp & 3;
    const int kh = (warp - (kGatherWarps + 1)) >> 2;  // columns [32 kh, 32 kh + 32) of each tile
    const int h = quarter * 32 + lane;                // head == TMEM lane
    const uint32_t tl = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    const bool leader = (h == 0 && kh == 0);          // re-arms the receive buffer
    {
      // this CTA's columns of q[r, h, :] as packed bf16 pairs (element 2i in
      // the low half of column i); the quarter's two warps take half each
      // (a thread's loads are all issued ahead of its tensor-memory stores:
      // a store is a compiler barrier, and loads issued one chunk at a time
      // would put five memory round trips before the first MMA)
      const uint16_t* qrow = P.q + (static_cast<int64_t>(r) * kH + h) * kDqk;
      constexpr int kChunks = kQk / 32;           // 32-column chunks: latent 0..7, rope 8
      constexpr int kMine = (kChunks + 1) / 2;    // chunks of the first warp of a quarter (the second: one fewer)
      const int c0 = kh == 0 ? 0 : kMine;
      const int nmine = kh == 0 ? kMine : kChunks - kMine;
      constexpr int kBatch = kMine;  // chunks whose loads are in flight together
#pragma unroll
      for (int i0 = 0; i0 < kMine; i0 += kBatch) {
        uint4 x[kBatch][4];
#pragma unroll
        for (int j = 0; j < kBatch; ++j) {
          const int i = i0 + j, c = c0 + i;
          const uint4* qs = reinterpret_cast<const uint4*>(qrow + (c < kLatCols / 32 ? a0 * 64 + c * 32 : rope0));
#pragma unroll
          for (int v = 0; v < 4; ++v) x[j][v] = i < nmine ? __ldg(qs + v) : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int j = 0; j < kBatch; ++j) {
          const int i = i0 + j;
          if (i >= nmine) break;
          uint32_t u[16];
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            u[4 * v + 0] = x[j][v].x;
            u[4 * v + 1] = x[j][v].y;
            u[4 * v + 2] = x[j][v].z;
            u[4 * v + 3] = x[j][v].w;
          }
          tmem_st16(tl + kQCol + (c0 + i) * 16, u);
        }
      }
      tmem_st_wait();
      tc_fence_before_sync();
      mbar_arrive(q_ready);
    }
    const uint32_t xin = sbase + kOffXin, xout = sbase + kOffXout;
    bool ok = true;
    float sreg[32], snext[32];
    float m_run = -INFINITY, l_half = 0.f;
    // S(t): this thread's 32 columns, then S(t) may be overwritten
    auto read_s = [&](float* dst) {
      tc_fence_after_sync();
      tmem_ld32(tl + kSCol + 32 * kh, dst);
      tc_fence_before_sync();
      mbar_arrive(s_empty);
    };
    // this thread's partial of the tile, chunk-major [16 x 4 rows][128 heads]
    auto write_x = [&](const float* v) {
#pragma unroll
      for (int c = 0; c < 8; ++c)
        asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(xout + ((kh * 8 + c) * kH + h) * 16),
                     "f"(v[4 * c]), "f"(v[4 * c + 1]), "f"(v[4 * c + 2]), "f"(v[4 * c + 3])
                     : "memory");
      fence_proxy_async_smem();  // generic writes -> bulk-copy reads
      mbar_arrive(xout_written);
    };
    // validity of this lane's row in tiles [j0, j0 + 32): the 32 list entries
    // are loaded together (one memory round trip), the first batch before
    // the wait for tile 0's logits, where it overlaps the first gather
    auto load_valid = [&](int j0) {
      int ix[32];
#pragma unroll
      for (int t = 0; t < 32; ++t) {
        const int rr = (j0 + t) * kRows + kh * 32 + lane;
        ix[t] = (j0 + t < T && rr < nrows) ? __ldg(sel + rr) : -1;
      }
      uint32_t bits = 0;
#pragma unroll
      for (int t = 0; t < 32; ++t) bits |= ((ix[t] >= 0 && ix[t] < L) ? 1u : 0u) << t;
      return bits;
    };
    uint32_t vbits = load_valid(0);
    int vbase = 0;
    if (T > 0) {
      if (!mbar_wait_warp(s_full, 0, abort_flag, P.err)) {
        ok = false;
      } else {
        read_s(sreg);
        write_x(sreg);
      }
    }
    for (int j = 0; ok && j < T; ++j) {
      const int bb = j & 1;
      if (j >= vbase + 32) {
        vbase = j;
        vbits = load_valid(j);
      }
      const uint32_t valid = __ballot_sync(0xffffffffu, ((vbits >> (j - vbase)) & 1u) != 0);
      // tile j + 1's partial goes out first, from every warp at the same
      // point, so its copy runs while this CTA waits for the other CTA's
      // partial of tile j and under this tile's softmax (tile j depends on
      // the other CTA's tiles j - 1 and j - 2 only)
      if (j + 1 < T) {
        if (!mbar_wait_warp(s_full, (j + 1) & 1, abort_flag, P.err)) { ok = false; break; }
        read_s(snext);
        // the copy of tile j has read xout
        if (!mbar_wait_warp(xout_free, j & 1, abort_flag, P.err)) { ok = false; break; }
        write_x(snext);
      }
      // S = S_0 + S_1
      if (!mbar_wait_warp_cluster(x_full(bb), (j >> 1) & 1, abort_flag, P.err)) { ok = false; break; }
      // arm for tile j + 2 (the other CTA sends it only after x_empty of tile j)
      if (leader && j + 2 < T) mbar_arrive_expect_tx(x_full(bb), kXBytes);
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const float4 v = ld_shared_v4f(xin + bb * kXBytes + ((kh * 8 + c) * kH + h) * 16);
        sreg[4 * c] += v.x;
        sreg[4 * c + 1] += v.y;
        sreg[4 * c + 2] += v.z;
        sreg[4 * c + 3] += v.w;
      }
      mbar_arrive(xin_read(bb));
      float mt = -INFINITY;
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const bool v = ((valid >> i) & 1u) != 0;
        sreg[i] = v ? sreg[i] * P.scale_log2 : -INFINITY;
        mt = fmaxf(mt, sreg[i]);
      }
      // tile max over all 64 columns: swap with the head's other warp
      const uint32_t red = sbase + kOffRed + bb * (2 * kH * 4);
      st_shared_f32(red + (kh * kH + h) * 4, mt);
      mbar_arrive(red_full(bb));
      if (!mbar_wait_warp(red_full(bb), (j >> 1) & 1, abort_flag, P.err)) { ok = false; break; }
      mt = fmaxf(mt, ld_shared_f32(red + ((kh ^ 1) * kH + h) * 4));
      // move the running max only when the tile max exceeds it by > 8 (base 2)
      const bool move = mt > m_run + 8.f;
      const bool rescale_o = move && m_run != -INFINITY;
      // O (and P in TMEM) hold tile j - 1's PV once it is done (PV of
      // tile j - 2 was awaited one tile ago, so the parity is unambiguous)
      if (j >= 1 && !mbar_wait_warp(pv_done, (j - 1) & 1, abort_flag, P.err)) { ok = false; break; }
      if (__any_sync(0xffffffffu, rescale_o)) {
        tc_fence_after_sync();
        rescale_o_cols(tl, kh * 128, kh * 128 + 128, rescale_o ? exp2f(m_run - mt) : 1.f);
      }
      if (move) {
        if (m_run != -INFINITY) l_half *= exp2f(m_run - mt);
        m_run = mt;
      }
      // P = 2^(s - m) in bf16 into TMEM (lane = head, column i = rows 2i, 2i+1
      // of this tile): the A operand of the value MMA
      float psum = 0.f;
      uint32_t pu[16];
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        const float p0 = (m_run == -INFINITY) ? 0.f : fast_exp2(sreg[2 * c] - m_run);
        const float p1 = (m_run == -INFINITY) ? 0.f : fast_exp2(sreg[2 * c + 1] - m_run);
        psum += p0 + p1;
        pu[c] = pack_bf16(p0, p1);
      }
      tmem_st16(tl + kPCol + 16 * kh, pu);
      tmem_st_wait();
      l_half += psum;
      tc_fence_before_sync();
      mbar_arrive(pv_ready);
#pragma unroll
      for (int i = 0; i < 32; ++i) sreg[i] = snext[i];
    }
    // final sum of head h: both warps' partial sums
    float m_fin = -INFINITY, l_fin = 0.f;
    if (ok && T > 0) {
      const uint32_t red_fin = sbase + kOffRed + (T & 1) * (2 * kH * 4);  // unused since tile T - 2
      st_shared_f32(red_fin + (kh * kH + h) * 4, l_half);
      mbar_arrive(fin);
      ok = mbar_wait_warp(fin, 0, abort_flag, P.err);
      if (ok) {
        m_fin = m_run;
        l_fin = l_half + ld_shared_f32(red_fin + ((kh ^ 1) * kH + h) * 4);
      }
    }
    // ------------------------------------------------------------ output --
    pdl_trigger();
    // (PV of tile T - 2 was awaited at tile T - 1: this parity is unambiguous)
    if (ok && T >= 1) ok = mbar_wait_warp(pv_done, (T - 1) & 1, abort_flag, P.err);
    if (ok) {
      tc_fence_after_sync();
      const int64_t rh = static_cast<int64_t>(r) * kH + h;
      const int c_lo = kh * 128, c_hi = c_lo + 128;
      // Each warp moves its 32 heads x 32 columns a chunk through its own
      // slot of the (now idle) ring: lane = head writes its row, then each
      // store instruction covers whole row segments (stores straight from
      // the lanes would touch 32 rows 1 KB apart per instruction).
      const uint32_t stage = sbase + kOffKV + (warp - (kGatherWarps + 1)) * kOutSlotBytes;
      const int h_w = quarter * 32;  // first head of this warp
      if (P.splits == 1) {
        const float inv = l_fin > 0.f ? 1.f / l_fin : 0.f;
        // bf16 row segment: 64 bytes, slot rows 80 bytes apart
        __nv_bfloat16* dst = P.out + (static_cast<int64_t>(r) * kH + h_w) * kDv + crank * kDvHalf;
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
            st_shared_u4(stage + lane * 80 + q * 16, v);
          }
          __syncwarp();
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int row = q * 8 + (lane >> 2), part = lane & 3;
            const uint4 v = ld_shared_u4(stage + row * 80 + part * 16);
            *reinterpret_cast<uint4*>(dst + static_cast<int64_t>(row) * kDv + c + part * 8) = v;
          }
          __syncwarp();
        }
        if (P.lse != nullptr && crank == 0 && kh == 0)
          P.lse[rh] = l_fin > 0.f ? (m_fin + log2f(l_fin)) * 0.6931471805599453f : -INFINITY;
      } else {
        const int64_t it = (static_cast<int64_t>(r) * P.splits + sp) * 2 + crank;
        // fp32 row segment: 128 bytes, slot rows 144 bytes apart
        float* dst = P.part_o + (it * kH + h_w) * kDvHalf;
#pragma unroll 1
        for (int c = c_lo; c < c_hi; c += 32) {
          float o[32];
          if (T >= 1) tmem_ld32(tl + c, o);
          else
            for (int i = 0; i < 32; ++i) o[i] = 0.f;
#pragma unroll
          for (int q = 0; q < 8; ++q)
            st_shared_u4(stage + lane * 144 + q * 16,
                         make_uint4(__float_as_uint(o[q * 4]), __float_as_uint(o[q * 4 + 1]),
                                    __float_as_uint(o[q * 4 + 2]), __float_as_uint(o[q * 4 + 3])));
          __syncwarp();
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            const int row = q * 4 + (lane >> 3), part = lane & 7;
            const uint4 v = ld_shared_u4(stage + row * 144 + part * 16);
            *reinterpret_cast<uint4*>(dst + row * kDvHalf + c + part * 4) = v;
          }
          __syncwarp();
        }
        if (crank == 0 && kh == 0) {
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
// kS = the split count, a template argument so that every load of a thread
// (four output positions x kS splits) is issued before the first is used.
template <int kS>
__global__ void __launch_bounds__(256) attn_combine_kernel(const float* __restrict__ part_o,
                                                           const float* __restrict__ part_ml,
                                                           __nv_bfloat16* __restrict__ out, float* __restrict__ lse) {
  constexpr int splits = kS;
  constexpr int kBatch = kS < 8 ? kS : 8;  // splits whose loads are in flight together
  pdl_wait();
  __shared__ float coef[kMaxSplits][kCombineHeads];
  const int r = blockIdx.x;
  const int h0 = blockIdx.y * kCombineHeads;
  const int tid = threadIdx.x;
  constexpr int kItr = kCombineHeads * (kDv / 4) / 256;  // output positions a thread
  auto load_batch = [&](int i0, float4 (&o)[kItr][kBatch]) {
#pragma unroll
    for (int itr = 0; itr < kItr; ++itr) {
      const int x = itr * 256 + tid;
      const int h = h0 + x / (kDv / 4);
      const int c4 = x % (kDv / 4);
      const int hv = c4 / (kDvHalf / 4);
      const int cc = (c4 % (kDvHalf / 4)) * 4;
#pragma unroll
      for (int i = 0; i < kBatch; ++i) {
        if (i0 + i < kS) {
          const int64_t it = (static_cast<int64_t>(r) * splits + i0 + i) * 2 + hv;
          o[itr][i] = __ldg(reinterpret_cast<const float4*>(part_o + (it * kH + h) * kDvHalf + cc));
        }
      }
    }
  };
  // the first batch of partial outputs is loaded before the weights are
  // formed (it does not depend on them), so the two overlap
  float4 o[kItr][kBatch];
  load_batch(0, o);
  if (tid < kCombineHeads) {
    const int h = h0 + tid;
    float M = -INFINITY;
    for (int i = 0; i < kS; ++i) {
      const int64_t it = static_cast<int64_t>(r) * splits + i;
      const float m = part_ml[(it * 2 + 0) * kH + h];
      const float l = part_ml[(it * 2 + 1) * kH + h];
      if (l > 0.f) M = fmaxf(M, m);
    }
    float Ls = 0.f;
    for (int i = 0; i < kS; ++i) {
      const int64_t it = static_cast<int64_t>(r) * splits + i;
      const float m = part_ml[(it * 2 + 0) * kH + h];
      const float l = part_ml[(it * 2 + 1) * kH + h];
      const float wgt = (l > 0.f) ? exp2f(m - M) : 0.f;
      coef[i][tid] = wgt;
      Ls += wgt * l;
    }
    const float inv = Ls > 0.f ? 1.f / Ls : 0.f;
    for (int i = 0; i < kS; ++i) coef[i][tid] *= inv;
    if (lse != nullptr)
      lse[static_cast<int64_t>(r) * kH + h] = Ls > 0.f ? (M + log2f(Ls)) * 0.6931471805599453f : -INFINITY;
  }
  __syncthreads();
  float4 acc[kItr];
#pragma unroll
  for (int itr = 0; itr < kItr; ++itr) acc[itr] = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
  for (int i0 = 0; i0 < kS; i0 += kBatch) {
    if (i0 > 0) load_batch(i0, o);
#pragma unroll
    for (int itr = 0; itr < kItr; ++itr) {
      const int hl = (itr * 256 + tid) / (kDv / 4);
#pragma unroll
      for (int i = 0; i < kBatch; ++i) {
        if (i0 + i < kS) {
          const float c = coef[i0 + i][hl];
          acc[itr].x = fmaf(c, o[itr][i].x, acc[itr].x);
          acc[itr].y = fmaf(c, o[itr][i].y, acc[itr].y);
          acc[itr].z = fmaf(c, o[itr][i].z, acc[itr].z);
          acc[itr].w = fmaf(c, o[itr][i].w, acc[itr].w);
        }
      }
    }
  }
#pragma unroll
  for (int itr = 0; itr < kItr; ++itr) {
    const int x = itr * 256 + tid;
    const int h = h0 + x / (kDv / 4);
    const int c4 = x % (kDv / 4);
    uint2 v;
    v.x = pack_bf16(acc[itr].x, acc[itr].y);
    v.y = pack_bf16(acc[itr].z, acc[itr].w);
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
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1] = pdl_attribute();
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  if (cudaLaunchKernelEx(&cfg, attn_mla_tc_kernel, P) != cudaSuccess) return DSA_ERR_CUDA;
  if (p.splits > 1) {
    cudaLaunchConfig_t cc = {};
    cc.gridDim = dim3(static_cast<unsigned>(R), kH / kCombineHeads, 1);
    cc.blockDim = dim3(256, 1, 1);
    cc.stream = a.stream;
    cudaLaunchAttribute cattr[1] = {pdl_attribute()};
    cc.attrs = cattr;
    cc.numAttrs = 1;
    cudaError_t e = cudaErrorInvalidValue;
    const float* po = P.part_o;
    const float* pm = P.part_ml;
    switch (p.splits) {
#define DSA_COMBINE_CASE(S) \
  case S: e = cudaLaunchKernelEx(&cc, attn_combine_kernel<S>, po, pm, P.out, a.lse); break;
      DSA_COMBINE_CASE(2) DSA_COMBINE_CASE(3) DSA_COMBINE_CASE(4) DSA_COMBINE_CASE(5) DSA_COMBINE_CASE(6)
      DSA_COMBINE_CASE(7) DSA_COMBINE_CASE(8) DSA_COMBINE_CASE(9) DSA_COMBINE_CASE(10) DSA_COMBINE_CASE(11)
      DSA_COMBINE_CASE(12) DSA_COMBINE_CASE(13) DSA_COMBINE_CASE(14) DSA_COMBINE_CASE(15) DSA_COMBINE_CASE(16)
#undef DSA_COMBINE_CASE
      default: return DSA_ERR_UNSUPPORTED;
    }
    if (e != cudaSuccess) return DSA_ERR_CUDA;
  }
  return DSA_OK;
}

}  // namespace dsa
