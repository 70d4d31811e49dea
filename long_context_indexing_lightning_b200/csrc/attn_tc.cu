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
// CTA 1 owns [256, 576).  Each CTA
//   * gathers only its own columns of the selected rows (cp.async, 16 bytes a
//     thread, into a 3-stage ring of 64-row tiles in the 128-byte-swizzled
//     K-major layout the MMA reads; padding and out-of-range rows are zero
//     filled),
//   * keeps its columns of Q in tensor memory (A operand of the logits MMA),
//   * computes its partial logits S_c = Q_c K_c^T (M = 128 heads, N = 64 rows),
//   * swaps partials with the other CTA (a bulk copy of 32 KB into the other
//     CTA's shared memory, completing on its barrier), so
//     both hold the same S = S_0 + S_1 (fp32 addition is commutative, so the
//     two sums are bit-identical) and run the same online softmax,
//   * accumulates its 256-column half of the output, O_c += P V_c, in TMEM
//     (V_0 = latent columns [0, 256), V_1 = [256, 512): each CTA's value half
//     lies inside the columns it already gathered).
// Warps: 0-3 gather, 4 issues tcgen05.mma, 5-8 (thread = head = TMEM lane)
// load Q into TMEM and run the softmax in base 2 with a running max that only
// moves (and O is rescaled in TMEM) when a tile max exceeds it by more than 8.
// Long selections are split across clusters and merged by a small combine
// kernel (log-sum-exp weights).  Every wait is bounded.
#include "dsa_common.cuh"
#include "dsa_internal.h"

namespace dsa {
namespace {

constexpr int kH = 128;                  // heads == MMA M
constexpr int kDqk = 576;                // latent 512 + rope 64
constexpr int kDv = 512;
constexpr int kDvHalf = 256;
constexpr int kRows = 64;                // selected rows per tile (MMA N of S, K of PV)
constexpr int kSplitCol = 256;           // CTA 0: columns [0, 256); CTA 1: [256, 576)
constexpr int kAtomsMax = 5;             // 64-column swizzle atoms per CTA (CTA 0 uses 4)
constexpr int kAtomBytes = kRows * 128;  // one atom of one tile: 8 KB
constexpr int kStageBytes = kAtomsMax * kAtomBytes;  // 40 KB
constexpr int kStages = 3;
constexpr int kGatherWarps = 4;
constexpr int kMmaWarp = 4;
constexpr int kSoftThreads = 128;
constexpr int kThreads = 32 * kGatherWarps + 32 + kSoftThreads;  // 288
// tensor memory: O half [0, 256), Q columns [256, 256 + 160), S [416, 480)
constexpr int kTmemCols = 512;
constexpr int kQCol = 256;
constexpr int kSCol = 416;

// shared memory map (from a 1024-aligned base)
constexpr int kOffKV = 0;
constexpr int kOffP = kOffKV + kStages * kStageBytes;  // P: 128 heads x 64 rows bf16, SW128 K-major
// partial logits, chunk-major [16 x 4 rows][128 heads] fp32: the other CTA's
// (received by bulk copy) and this CTA's (sent from here)
constexpr int kXBytes = kH * kRows * 4;
constexpr int kOffXin = kOffP + kH * kRows * 2;
constexpr int kOffXout = kOffXin + kXBytes;
constexpr int kOffBar = kOffXout + kXBytes;
// barriers: kv_full[3], kv_empty[3], s_full, s_empty, p_full, p_empty, o_done,
//           q_ready, x_full, x_empty, mma_done, xout_free, xout_written, xin_read
constexpr int kNumBars = 2 * kStages + 12;
constexpr int kOffMisc = kOffBar + kNumBars * 8;
constexpr int kSmemBytes = kOffMisc + 16 + 1024;

struct AttnParams {
  const uint16_t* q;        // [R][128][576] bf16
  const uint16_t* kv;       // [B][s_max][576] bf16
  const int32_t* idx;       // [R][k]
  const int32_t* ctx_len;   // [B]
  __nv_bfloat16* out;       // [R][128][512]
  float* lse;               // [R][128] or null
  float* part_o;            // [R][S][2][128][256] (splits > 1)
  float* part_ml;           // [R][S][2][2][128]: m then l (splits > 1)
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
__device__ __forceinline__ void st_cluster_v4f(uint32_t raddr, float a, float b, float c, float d) {
  asm volatile("st.shared::cluster.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(raddr), "f"(a), "f"(b), "f"(c), "f"(d)
               : "memory");
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

__global__ void __launch_bounds__(kThreads, 1) attn_mla_tc_kernel(AttnParams P) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_addr(smem);
  const uint32_t bar0 = sbase + kOffBar;
  auto kv_full = [&](int i) { return bar0 + 8u * i; };
  auto kv_empty = [&](int i) { return bar0 + 8u * (kStages + i); };
  const uint32_t s_full = bar0 + 8u * (2 * kStages + 0);
  const uint32_t s_empty = bar0 + 8u * (2 * kStages + 1);
  const uint32_t p_full = bar0 + 8u * (2 * kStages + 2);
  const uint32_t p_empty = bar0 + 8u * (2 * kStages + 3);
  const uint32_t o_done = bar0 + 8u * (2 * kStages + 4);
  const uint32_t q_ready = bar0 + 8u * (2 * kStages + 5);
  const uint32_t x_full = bar0 + 8u * (2 * kStages + 6);
  const uint32_t x_empty = bar0 + 8u * (2 * kStages + 7);
  const uint32_t mma_done = bar0 + 8u * (2 * kStages + 8);
  const uint32_t xout_free = bar0 + 8u * (2 * kStages + 9);
  const uint32_t xout_written = bar0 + 8u * (2 * kStages + 10);
  const uint32_t xin_read = bar0 + 8u * (2 * kStages + 11);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffMisc + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = lane_id();
  const uint32_t crank = cluster_rank();  // 0: latent columns [0, 256); 1: [256, 576)
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
    mbar_init(s_full, 1);
    mbar_init(s_empty, kSoftThreads);
    mbar_init(p_full, kSoftThreads);
    mbar_init(p_empty, 1);
    mbar_init(o_done, 1);
    mbar_init(q_ready, kSoftThreads);
    mbar_init(x_full, 1);   // own arm (expect_tx) + the other CTA's bulk copy
    mbar_init(x_empty, 1);  // arrived by the other CTA once it has read our partial
    mbar_init(mma_done, 1);
    mbar_init(xout_free, 1);
    mbar_init(xout_written, kSoftThreads);
    mbar_init(xin_read, kSoftThreads);
    if (T > 0) mbar_arrive_expect_tx(x_full, kXBytes);  // armed for tile 0
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(smem_addr(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  cluster_sync_all();  // both CTAs' barriers exist before any remote arrival
  const uint32_t tmem = *tmem_slot;

  if (warp < kGatherWarps) {
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
        // O += P(np) V(np) as soon as P is written (frees the tile's stage)
        if (np < nq && mbar_test_wait(p_full, np & 1)) {
          tc_fence_after_sync();
          const uint64_t st_off = static_cast<uint64_t>(((np % kStages) * kStageBytes) >> 4);
#pragma unroll
          for (int kk = 0; kk < kRows / 16; ++kk)
            tc_mma_f16(tmem, p_desc0 + ((kk * 32) >> 4), v_desc0 + st_off + ((kk * 16 * 128) >> 4), idesc_o,
                       (np > 0 || kk > 0) ? 1u : 0u);
          tc_commit(kv_empty(np % kStages));
          tc_commit(p_empty);
          tc_commit(o_done);
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
  } else {
    // ------------------------------------- Q to TMEM, softmax, output --
    const int quarter = warp & 3;
    const int h = quarter * 32 + lane;  // head == TMEM lane
    const uint32_t tl = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    {
      // this CTA's columns of q[r, h, :] as packed bf16 pairs (element 2i in
      // the low half of column i)
      const uint4* qs = reinterpret_cast<const uint4*>(P.q + (static_cast<int64_t>(r) * kH + h) * kDqk + a0 * 64);
      for (int c = 0; c < natoms * 64 / 32; ++c) {
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
    const uint32_t xin = sbase + kOffXin, xout = sbase + kOffXout;
    const uint32_t xin_peer = map_peer(xin, peer);
    const uint32_t x_full_peer = map_peer(x_full, peer);
    const uint32_t x_empty_peer = map_peer(x_empty, peer);
    const bool leader = (h == 0);  // issues the bulk copy and the cross-CTA signals
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    int nx0 = (lane < nrows) ? __ldg(sel + lane) : -1;
    int nx1 = (lane + 32 < nrows) ? __ldg(sel + lane + 32) : -1;
    for (int j = 0; j < T; ++j) {
      // which rows of this tile are real (indices fetched one tile ahead)
      const uint32_t valid0 = __ballot_sync(0xffffffffu, nx0 >= 0 && nx0 < L);
      const uint32_t valid1 = __ballot_sync(0xffffffffu, nx1 >= 0 && nx1 < L);
      const int jn = (j + 1) * kRows + lane;
      nx0 = (j + 1 < T && jn < nrows) ? __ldg(sel + jn) : -1;
      nx1 = (j + 1 < T && jn + 32 < nrows) ? __ldg(sel + jn + 32) : -1;
      if (!mbar_wait_warp(s_full, j & 1, abort_flag, P.err)) { ok = false; break; }
      tc_fence_after_sync();
      float s[kRows];
      tmem_ld32(tl + kSCol, s);
      tmem_ld32(tl + kSCol + 32, s + 32);
      tc_fence_before_sync();
      mbar_arrive(s_empty);
      // swap partial logits with the other CTA: stage mine locally, one
      // thread copies the 32 KB into the other CTA's receive buffer ...
      if (leader && j >= 1) {
        asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");  // previous copy has read xout
        mbar_arrive(xout_free);
      }
      if (!mbar_wait_warp(xout_free, (j & 1) ^ 1, abort_flag, P.err)) { ok = false; break; }
#pragma unroll
      for (int c = 0; c < kRows / 4; ++c)
        asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(xout + (c * kH + h) * 16), "f"(s[4 * c]),
                     "f"(s[4 * c + 1]), "f"(s[4 * c + 2]), "f"(s[4 * c + 3])
                     : "memory");
      fence_proxy_async_smem();
      mbar_arrive(xout_written);
      if (leader) {
        bool go = mbar_wait(xout_written, j & 1, abort_flag, P.err);
        if (go && j >= 1) {
          // the other CTA has read our previous partial
          go = false;
          const uint64_t t0 = global_timer_ns();
          for (uint32_t it = 0; it < kWaitLimitPolls; ++it) {
            if (mbar_try_wait_cluster(x_empty, (j - 1) & 1)) { go = true; break; }
            if ((it & 63u) == 63u && (*abort_flag || global_timer_ns() - t0 > kWaitLimitNs)) break;
          }
          if (!go && !*abort_flag) { *abort_flag = 1; raise_error(P.err, kErrTimeout); }
        }
        if (go) {
          asm volatile(
              "cp.async.bulk.shared::cluster.shared::cta.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n\t"
              "cp.async.bulk.commit_group;" ::"r"(xin_peer),
              "r"(xout), "r"(kXBytes), "r"(x_full_peer)
              : "memory");
        }
      }
      // ... and the other CTA's partial arrives in ours: S = S_0 + S_1 on both sides
      if (!mbar_wait_warp_cluster(x_full, j & 1, abort_flag, P.err)) { ok = false; break; }
#pragma unroll
      for (int c = 0; c < kRows / 4; ++c) {
        const float4 v = ld_shared_v4f(xin + (c * kH + h) * 16);
        s[4 * c] += v.x;
        s[4 * c + 1] += v.y;
        s[4 * c + 2] += v.z;
        s[4 * c + 3] += v.w;
      }
      mbar_arrive(xin_read);
      if (leader) {
        if (mbar_wait(xin_read, j & 1, abort_flag, P.err)) {
          if (j + 1 < T) mbar_arrive_expect_tx(x_full, kXBytes);  // arm for the next tile
          mbar_arrive_remote(x_empty_peer);
        }
      }
      float mt = -INFINITY;
#pragma unroll
      for (int i = 0; i < kRows; ++i) {
        const bool v = ((i < 32 ? (valid0 >> i) : (valid1 >> (i - 32))) & 1u) != 0;
        s[i] = v ? s[i] * P.scale_log2 : -INFINITY;
        mt = fmaxf(mt, s[i]);
      }
      // move the running max only when the tile max exceeds it by > 8 (base 2)
      const bool move = mt > m_run + 8.f;
      const bool rescale_o = move && m_run != -INFINITY;
      if (__any_sync(0xffffffffu, rescale_o)) {
        // O must hold every previous tile before it is rescaled
        if (j >= 1 && !mbar_wait_warp(o_done, (j - 1) & 1, abort_flag, P.err)) { ok = false; break; }
        tc_fence_after_sync();
        const float f = rescale_o ? exp2f(m_run - mt) : 1.f;
#pragma unroll 1
        for (int c = 0; c < kDvHalf; c += 32) {
          float o[32];
          tmem_ld32(tl + c, o);
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] *= f;
          tmem_st32f(tl + c, o);
        }
        tmem_st_wait();
      }
      if (move) {
        if (m_run != -INFINITY) l_run *= exp2f(m_run - mt);
        m_run = mt;
      }
      // P = 2^(s - m) in bf16: one 128-byte row per head, 128-byte-swizzled K-major
      if (j >= 1 && !mbar_wait_warp(p_empty, (j - 1) & 1, abort_flag, P.err)) { ok = false; break; }
      const uint32_t prow = sbase + kOffP + (h >> 3) * 1024 + (h & 7) * 128;
      float psum = 0.f;
#pragma unroll
      for (int c = 0; c < kRows / 8; ++c) {
        float p[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          p[e] = (m_run == -INFINITY) ? 0.f : fast_exp2(s[c * 8 + e] - m_run);
          psum += p[e];
        }
        st_shared_v4(prow + ((c ^ (h & 7)) << 4), pack_bf16(p[0], p[1]), pack_bf16(p[2], p[3]),
                     pack_bf16(p[4], p[5]), pack_bf16(p[6], p[7]));
      }
      l_run += psum;
      fence_proxy_async_smem();
      tc_fence_before_sync();
      mbar_arrive(p_full);
    }
    if (leader) asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
    // ------------------------------------------------------------ output --
    if (ok && T >= 1) ok = mbar_wait_warp(o_done, (T - 1) & 1, abort_flag, P.err);
    if (ok) {
      tc_fence_after_sync();
      const int64_t rh = static_cast<int64_t>(r) * kH + h;
      if (P.splits == 1) {
        const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
        __nv_bfloat16* dst = P.out + rh * kDv + crank * kDvHalf;
#pragma unroll 1
        for (int c = 0; c < kDvHalf; c += 32) {
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
        if (P.lse != nullptr && crank == 0)
          P.lse[rh] = l_run > 0.f ? (m_run + log2f(l_run)) * 0.6931471805599453f : -INFINITY;
      } else {
        const int64_t it = (static_cast<int64_t>(r) * P.splits + sp) * 2 + crank;
        float* dst = P.part_o + (it * kH + h) * kDvHalf;
#pragma unroll 1
        for (int c = 0; c < kDvHalf; c += 32) {
          float o[32];
          if (T >= 1) tmem_ld32(tl + c, o);
          else
            for (int i = 0; i < 32; ++i) o[i] = 0.f;
#pragma unroll
          for (int q = 0; q < 8; ++q)
            *reinterpret_cast<float4*>(dst + c + q * 4) = make_float4(o[q * 4], o[q * 4 + 1], o[q * 4 + 2], o[q * 4 + 3]);
        }
        P.part_ml[(it * 2 + 0) * kH + h] = m_run;
        P.part_ml[(it * 2 + 1) * kH + h] = l_run;
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
      const int64_t it = (static_cast<int64_t>(r) * splits + i) * 2;
      const float m = part_ml[(it * 2 + 0) * kH + h];
      const float l = part_ml[(it * 2 + 1) * kH + h];
      if (l > 0.f) M = fmaxf(M, m);
    }
    float Ls = 0.f;
    for (int i = 0; i < splits; ++i) {
      const int64_t it = (static_cast<int64_t>(r) * splits + i) * 2;
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
