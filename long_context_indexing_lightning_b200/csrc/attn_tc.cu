// Sparse MLA attention over the selected latent rows, on the tensor cores.
//
// DeepSeek-V3.2 model doc (Transformers), section "DeepSeek Sparse Attention
// (DSA)", item 2: main MLA attention runs only over the index_topk tokens the
// indexer kept, O(index_topk) per query instead of O(L).  Absorbed (MQA) form
// of MLA (section DeepseekV32Config: num_attention_heads 128, kv_lora_rank
// 512, qk_rope_head_dim 64): every head's 576-wide query meets one shared
// 576-wide latent row per token; the value is the row's first 512 columns.
//
// One CTA = (query row, split of its selected list, half of d_v).
//   * The output of one query (128 heads x 512 fp32) would fill all of tensor
//     memory, so a CTA accumulates one 256-column half of it in TMEM; the
//     two halves recompute the same logits (S = Q K^T, M = 128 heads).
//   * Warps 0-3 gather the selected latent rows (1152 bytes each) into a
//     2-stage shared-memory ring with TMA row gathers (tile::gather4, four
//     rows x 64 columns per instruction) into the 128-byte-swizzled K-major
//     layout the MMA reads; padding (-1) or out-of-range rows are read at
//     row -1, which TMA fills with zeros.
//   * Warp 4 loads Q once with TMA and issues tcgen05.mma: S(j) for tile j
//     (32 rows) in three chunks, and O += P(j-1) V(j-1) as soon as P is ready
//     (between chunks if need be), so the logits of the next tile are
//     computed while the softmax warps work on the current one.
//   * Warps 5-8 (thread = head = TMEM lane) run the online softmax in base 2:
//     read S, mask, keep a running max that is only moved (and O rescaled in
//     TMEM) when the tile max exceeds it by more than 2^8, write P as bf16
//     into the part of the tile's stage that the value half does not use, and
//     finally normalise O (or store an unnormalised partial for the split
//     combine).
#include "dsa_common.cuh"
#include "dsa_internal.h"

namespace dsa {
namespace {

constexpr int kH = 128;                 // heads == MMA M
constexpr int kDqk = 576;               // latent 512 + rope 64
constexpr int kDv = 512;
constexpr int kDvHalf = 256;
constexpr int kRows = 32;               // selected rows per tile (MMA N of S, K of PV)
constexpr int kKB = kDqk / 64;          // 9 swizzle atoms of 64 columns
constexpr int kBox = kRows * 128;       // bytes of one 64-column block of a tile (4 KB)
constexpr int kTile = kKB * kBox;       // 36 KB
constexpr int kQBytes = kKB * kH * 128; // 144 KB
constexpr int kStages = 2;
constexpr int kSoftThreads = 128;
constexpr int kGatherWarps = 4;
constexpr int kMmaWarp = kGatherWarps;
constexpr int kThreads = 32 * kGatherWarps + 32 + kSoftThreads;  // gather warps, MMA warp, 4 softmax warps
constexpr int kTmemCols = 512;          // O half: cols [0,256), S buffers: [256,288), [288,320)
constexpr int kSCol = 256;

// shared memory map (from a 1024-aligned base)
constexpr int kOffQ = 0;
constexpr int kOffKV = kOffQ + kQBytes;
constexpr int kOffBar = kOffKV + kStages * kTile;
// barriers: kv_full[2], kv_empty[2], s_full[2], s_empty[2], p_full[2], o_done, q_full, mma_done
constexpr int kNumBars = 13;
constexpr int kOffMisc = kOffBar + kNumBars * 8;
constexpr int kSmemBytes = kOffMisc + 16 + 1024;

struct AttnParams {
  const uint16_t* kv;       // [B][s_max][576] bf16
  const int32_t* idx;       // [R][k]
  const int32_t* ctx_len;   // [B]
  __nv_bfloat16* out;       // [R][128][512]
  float* lse;               // [R][128] or null
  float* part_o;            // [R][S][2][128][256] (splits > 1)
  float* part_ml;           // [R][S][2][128] : m then l (splits > 1)
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
constexpr uint32_t kLayoutSW128 = 2, kLayoutSW64 = 4;

// kind::f16 instruction descriptor with B stored MN-major (N contiguous).
__host__ __device__ constexpr uint32_t idesc_bf16_f32_bmn(int M, int N) {
  return idesc_bf16_f32(M, N) | (1u << 16);
}

// TMA row gather: rows r0..r3 of a 2-D tensor map, 64 columns from `col`,
// written as four consecutive 128-byte swizzled rows at `dst`.
__device__ __forceinline__ void tma_gather4(uint32_t dst, const CUtensorMap* map, uint32_t bar, int col, int r0,
                                            int r1, int r2, int r3) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile::gather4.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4, %5, %6}], [%7];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(col), "r"(r0), "r"(r1), "r"(r2), "r"(r3), "r"(bar)
      : "memory");
}
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
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
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float* v) {
  uint32_t u[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) u[i] = __float_as_uint(v[i]);
  tmem_st16(taddr, u);
#pragma unroll
  for (int i = 0; i < 16; ++i) u[i] = __float_as_uint(v[16 + i]);
  tmem_st16(taddr + 16, u);
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}


__global__ void __launch_bounds__(kThreads, 1)
    attn_mla_tc_kernel(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_kv,
                       AttnParams P) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_addr(smem);
  const uint32_t bar0 = sbase + kOffBar;
  auto kv_full = [&](int i) { return bar0 + 8u * i; };
  auto kv_empty = [&](int i) { return bar0 + 8u * (2 + i); };
  auto s_full = [&](int i) { return bar0 + 8u * (4 + i); };
  auto s_empty = [&](int i) { return bar0 + 8u * (6 + i); };
  auto p_full = [&](int i) { return bar0 + 8u * (8 + i); };
  const uint32_t o_done = bar0 + 8u * 10;
  const uint32_t q_full = bar0 + 8u * 11;
  const uint32_t mma_done = bar0 + 8u * 12;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffMisc + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = lane_id();
  // work item
  const int hv = blockIdx.x & 1;
  const int sp = (blockIdx.x >> 1) % P.splits;
  const int r = (blockIdx.x >> 1) / P.splits;
  const int b = r / P.n_q;
  const int L = min(max(__ldg(P.ctx_len + b), 0), P.s_max);
  const int row0 = sp * P.rows_per_split;
  const int nrows = max(0, min(P.rows_per_split, P.k - row0));
  const int T = (nrows + kRows - 1) / kRows;
  const int32_t* sel = P.idx + static_cast<int64_t>(r) * P.k + row0;
  const uint32_t p_off = hv == 0 ? 4u * kBox : 0u;    // P lives where this half's V does not
  const uint32_t v_off = hv == 0 ? 0u : 4u * kBox;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(kv_full(i), kGatherWarps);
      mbar_init(kv_empty(i), 1);
      mbar_init(s_full(i), 1);
      mbar_init(s_empty(i), kSoftThreads);
      mbar_init(p_full(i), kSoftThreads);
    }
    mbar_init(o_done, 1);
    mbar_init(q_full, 1);
    mbar_init(mma_done, 1);
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
  const uint32_t tmem = *tmem_slot;

  if (warp < kGatherWarps) {
    // -------------------------------------------------- gather (TMA) --
    bool bad = false;
    // lane i holds the (flattened) row of tile row i; the next tile's
    // indices are fetched before this tile's gathers go out
    int nxt = (lane < nrows) ? __ldg(sel + lane) : -1;
    const int grp = lane & 7;  // this lane gathers rows 4*grp .. 4*grp+3
    for (int j = 0; j < T; ++j) {
      const int st = j & 1;
      int cur = nxt;
      if (cur >= L) { bad = true; cur = -1; }
      const int grow = cur >= 0 ? b * P.s_max + cur : -1;  // row -1 reads zeros
      const int jn = (j + 1) * kRows + lane;
      nxt = (j + 1 < T && jn < nrows) ? __ldg(sel + jn) : -1;
      const int r0 = __shfl_sync(0xffffffffu, grow, 4 * grp + 0);
      const int r1 = __shfl_sync(0xffffffffu, grow, 4 * grp + 1);
      const int r2 = __shfl_sync(0xffffffffu, grow, 4 * grp + 2);
      const int r3 = __shfl_sync(0xffffffffu, grow, 4 * grp + 3);
      if (!mbar_wait_warp(kv_empty(st), ((j >> 1) & 1) ^ 1, abort_flag, P.err)) break;
      // warp w gathers the 64-column blocks w, w+4, w+8 of the tile; each
      // warp's first lane adds its share of the bytes to the stage's barrier
      int nblk = 0;
      for (int kb = warp; kb < kKB; kb += kGatherWarps) ++nblk;
      if (lane == 0) mbar_arrive_expect_tx(kv_full(st), nblk * 8 * 512);
      __syncwarp();
      const uint32_t dst0 = sbase + kOffKV + st * kTile + grp * 512;
      for (int kb = warp + kGatherWarps * (lane >> 3); kb < kKB && (lane >> 3) < 3; kb += kGatherWarps * 4)
        tma_gather4(dst0 + kb * kBox, &tmap_kv, kv_full(st), kb * 64, r0, r1, r2, r3);
    }
    if (__any_sync(0xffffffffu, bad) && lane == 0) raise_error(P.err, kErrBadIndex);
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------- MMA issue --
    if (lane == 0) {
      const uint32_t qaddr = sbase + kOffQ;
      mbar_arrive_expect_tx(q_full, kQBytes);
#pragma unroll 1
      for (int kb = 0; kb < kKB; ++kb) tma_load_2d(qaddr + kb * kH * 128, &tmap_q, q_full, kb * 64, r * kH);
      constexpr uint32_t idesc_s = idesc_bf16_f32(kH, kRows);
      constexpr uint32_t idesc_o = idesc_bf16_f32_bmn(kH, kDvHalf);
      const uint64_t q_desc0 = sdesc(qaddr, 16, 1024, kLayoutSW128);
      const uint64_t kv_desc0 = sdesc(sbase + kOffKV, 16, 1024, kLayoutSW128);
      const uint64_t p_desc0 = sdesc(sbase + kOffKV + p_off, 16, 512, kLayoutSW64);
      const uint64_t v_desc0 = sdesc(sbase + kOffKV + v_off, kBox, 1024, kLayoutSW128);
      bool ok = mbar_wait(q_full, 0, abort_flag, P.err);
      auto do_pv = [&](int i) -> bool {
        if (!mbar_wait(p_full(i & 1), (i >> 1) & 1, abort_flag, P.err)) return false;
        tc_fence_after_sync();
        const uint64_t st_off = static_cast<uint64_t>(((i & 1) * kTile) >> 4);
#pragma unroll
        for (int kk = 0; kk < kRows / 16; ++kk)
          tc_mma_f16(tmem, p_desc0 + st_off + ((kk * 32) >> 4), v_desc0 + st_off + ((kk * 16 * 128) >> 4), idesc_o,
                     (i > 0 || kk > 0) ? 1u : 0u);
        tc_commit(kv_empty(i & 1));
        tc_commit(o_done);
        return true;
      };
      // Issue whichever of QK(nq) / PV(np) is ready (PV first), so the value
      // product of a tile -- which frees its stage for the next gather -- never
      // waits behind the logits of a tile whose rows are still in flight.
      // S(j) = Q K(j)^T is issued in kQkParts chunks; a P(i) that becomes
      // ready is issued between chunks, so the value product of a tile (which
      // frees its stage for the next gather) never queues behind a whole QK.
      constexpr int kQkMma = kDqk / 16;  // 36
      constexpr int kQkParts = 3;
      auto issue_qk_part = [&](int j, int part) {
        const int st = j & 1;
        if (part == 0) tc_fence_after_sync();
        const uint32_t d = tmem + kSCol + st * kRows;
        const uint64_t kv0 = kv_desc0 + static_cast<uint64_t>((st * kTile) >> 4);
#pragma unroll
        for (int q = 0; q < kQkMma / kQkParts; ++q) {
          const int kk = part * (kQkMma / kQkParts) + q;
          // descriptor start addresses advance in 16-byte units
          const uint32_t a_off = (kk >> 2) * kH * 128 + (kk & 3) * 32;
          const uint32_t b_off = (kk >> 2) * kBox + (kk & 3) * 32;
          tc_mma_f16(d, q_desc0 + (a_off >> 4), kv0 + (b_off >> 4), idesc_s, kk > 0 ? 1u : 0u);
        }
        if (part == kQkParts - 1) tc_commit(s_full(st));
      };
      int nq = 0, np = 0, qpart = 0;  // QK(nq) has issued qpart chunks
      uint64_t t0 = 0;
      uint32_t spins = 0;
      while (ok && np < T) {
        if (np < nq && mbar_test_wait(p_full(np & 1), (np >> 1) & 1)) {
          ok = do_pv(np);
          ++np;
          spins = 0;
          continue;
        }
        if (qpart > 0) {
          issue_qk_part(nq, qpart);
          if (++qpart == kQkParts) { qpart = 0; ++nq; }
          spins = 0;
          continue;
        }
        if (nq < T && mbar_test_wait(kv_full(nq & 1), (nq >> 1) & 1) &&
            mbar_test_wait(s_empty(nq & 1), ((nq >> 1) & 1) ^ 1)) {
          issue_qk_part(nq, 0);
          qpart = 1;
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
    // ------------------------------------------------ softmax + output --
    const int quarter = warp & 3;
    const int h = quarter * 32 + lane;                       // head == TMEM lane
    const uint32_t tl = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    int sidx_next = (lane < nrows) ? __ldg(sel + lane) : -1;
    for (int j = 0; j < T; ++j) {
      const int st = j & 1;
      // which rows of this tile are real (indices fetched one tile ahead)
      const int sidx = sidx_next;
      const int jn = (j + 1) * kRows + lane;
      sidx_next = (j + 1 < T && jn < nrows) ? __ldg(sel + jn) : -1;
      const uint32_t valid = __ballot_sync(0xffffffffu, sidx >= 0 && sidx < L);
      if (!mbar_wait_warp(s_full(st), (j >> 1) & 1, abort_flag, P.err)) { ok = false; break; }
      tc_fence_after_sync();
      float s[kRows];
      tmem_ld32(tl + kSCol + st * kRows, s);
      tc_fence_before_sync();
      mbar_arrive(s_empty(st));
      float mt = -INFINITY;
#pragma unroll
      for (int i = 0; i < kRows; ++i) {
        s[i] = ((valid >> i) & 1u) ? s[i] * P.scale_log2 : -INFINITY;
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
          tmem_st32(tl + c, o);
        }
        tmem_st_wait();
      }
      if (move) {
        if (m_run != -INFINITY) l_run *= exp2f(m_run - mt);
        m_run = mt;
      }
      // P = 2^(s - m) in bf16, 64 bytes per head, 64-byte-swizzled K-major
      const uint32_t prow = sbase + kOffKV + st * kTile + p_off + (h >> 3) * 512 + (h & 7) * 64;
      const int sw = (h >> 1) & 3;
      float psum = 0.f;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        float p[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          p[e] = (m_run == -INFINITY) ? 0.f : fast_exp2(s[c * 8 + e] - m_run);
          psum += p[e];
        }
        st_shared_v4(prow + ((c ^ sw) << 4), pack_bf16(p[0], p[1]), pack_bf16(p[2], p[3]), pack_bf16(p[4], p[5]),
                     pack_bf16(p[6], p[7]));
      }
      l_run += psum;
      fence_proxy_async_smem();
      tc_fence_before_sync();
      mbar_arrive(p_full(st));
    }
    // ------------------------------------------------------------ output --
    if (ok && T >= 1) ok = mbar_wait_warp(o_done, (T - 1) & 1, abort_flag, P.err);
    if (ok) {
      tc_fence_after_sync();
      const int64_t rh = static_cast<int64_t>(r) * kH + h;
      if (P.splits == 1) {
        const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
        __nv_bfloat16* dst = P.out + rh * kDv + hv * kDvHalf;
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
        if (P.lse != nullptr && hv == 0)
          P.lse[rh] = l_run > 0.f ? (m_run + log2f(l_run)) * 0.6931471805599453f : -INFINITY;
      } else {
        const int64_t item = (static_cast<int64_t>(r) * P.splits + sp) * 2 + hv;
        float* dst = P.part_o + (item * kH + h) * kDvHalf;
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
        P.part_ml[(item * 2 + 0) * kH + h] = m_run;
        P.part_ml[(item * 2 + 1) * kH + h] = l_run;
      }
    }
  }

  tc_fence_before_sync();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after_sync();
    tmem_dealloc(tmem, kTmemCols);
  }
}
}  // namespace
}  // namespace dsa

namespace dsa {
namespace {

constexpr int kMaxSplits = 16;

constexpr int kCombineHeads = 8;  // heads per combine block

// Merge the per-split partial outputs of each query: O = sum_i 2^(m_i - M) O_i
// / sum_i 2^(m_i - M) l_i with M = max_i m_i (base-2 log-sum-exp combine).
// Block = (query, group of 8 heads); 256 threads, 4 output columns each step.
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
      const int64_t item = (static_cast<int64_t>(r) * splits + i) * 2;
      const float m = part_ml[(item * 2 + 0) * kH + h];
      const float l = part_ml[(item * 2 + 1) * kH + h];
      if (l > 0.f) M = fmaxf(M, m);
    }
    float Ls = 0.f;
    for (int i = 0; i < splits; ++i) {
      const int64_t item = (static_cast<int64_t>(r) * splits + i) * 2;
      const float m = part_ml[(item * 2 + 0) * kH + h];
      const float l = part_ml[(item * 2 + 1) * kH + h];
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
  for (int it = 0; it < kCombineHeads * (kDv / 4) / 256; ++it) {
    const int x = it * 256 + tid;
    const int hl = x / (kDv / 4);
    const int c4 = x % (kDv / 4);
    const int h = h0 + hl;
    const int hv = c4 / (kDvHalf / 4);
    const int cc = (c4 % (kDvHalf / 4)) * 4;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int i = 0; i < splits; ++i) {
      const int64_t item = (static_cast<int64_t>(r) * splits + i) * 2 + hv;
      const float4 o = __ldg(reinterpret_cast<const float4*>(part_o + (item * kH + h) * kDvHalf + cc));
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

}  // namespace

bool attn_tc_supported(int H, int d_qk, int d_v, int KVH) {
  return H == kH && d_qk == kDqk && d_v == kDv && KVH == 1;
}

size_t attn_workspace_bytes(int B, int n_q, int H, int d_qk, int d_v, int KVH, int k, int dtype) {
  if (dtype != DSA_BF16 || !attn_tc_supported(H, d_qk, d_v, KVH)) return 0;
  const int64_t R = static_cast<int64_t>(B) * n_q;
  // the split plan depends on the SM count; size for the largest plan any
  // B200-class part (<= 256 SMs) would pick
  const SplitPlan p = plan_splits(R, k, 256);
  if (p.splits <= 1) return 0;
  const size_t items = static_cast<size_t>(R) * p.splits * 2;
  return items * kH * kDvHalf * 4 + items * 2 * kH * 4;
}

dsa_status_t attn_tc(const AttnArgs& a) {
  const int64_t R = static_cast<int64_t>(a.B) * a.n_q;
  if (R == 0) return DSA_OK;
  const int num_sms = device_sm_count(a.device);
  const SplitPlan p = plan_splits(R, a.k, num_sms);
  if (R * p.splits * 2 > INT32_MAX) return DSA_ERR_UNSUPPORTED;
  AttnParams P;
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
    const size_t items = static_cast<size_t>(R) * p.splits * 2;
    const size_t need = items * kH * kDvHalf * 4 + items * 2 * kH * 4;
    if (a.ws == nullptr || a.ws_bytes < need) return DSA_ERR_WORKSPACE;
    P.part_o = static_cast<float*>(a.ws);
    P.part_ml = P.part_o + items * kH * kDvHalf;
  }
  CUtensorMap tmq;
  if (!make_tmap_2d(&tmq, a.q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, kDqk, static_cast<uint64_t>(R) * kH, 64, kH))
    return DSA_ERR_CUDA;
  CUtensorMap tmkv;
  if (!make_tmap_2d(&tmkv, a.kv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, kDqk, static_cast<uint64_t>(a.B) * a.s_max, 64,
                    1))
    return DSA_ERR_CUDA;
  static bool attr_done[64] = {};
  if (a.device < 64 && !attr_done[a.device]) {
    if (cudaFuncSetAttribute(attn_mla_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes) !=
        cudaSuccess)
      return DSA_ERR_CUDA;
    attr_done[a.device] = true;
  }
  const unsigned grid = static_cast<unsigned>(R * p.splits * 2);
  attn_mla_tc_kernel<<<grid, kThreads, kSmemBytes, a.stream>>>(tmq, tmkv, P);
  if (cudaGetLastError() != cudaSuccess) return DSA_ERR_CUDA;
  if (p.splits > 1) {
    attn_combine_kernel<<<dim3(static_cast<unsigned>(R), kH / kCombineHeads), 256, 0, a.stream>>>(P.part_o, P.part_ml, p.splits, P.out,
                                                                       a.lse);
    if (cudaGetLastError() != cudaSuccess) return DSA_ERR_CUDA;
  }
  return DSA_OK;
}

}  // namespace dsa

namespace dsa {
// Exact scratch bytes the tensor-core attention needs for this shape on a
// device with `num_sms` SMs (0 when it writes its output directly).
size_t attn_scratch_bytes(int B, int n_q, int k, int num_sms) {
  const int64_t R = static_cast<int64_t>(B) * n_q;
  if (R == 0) return 0;
  const SplitPlan p = plan_splits(R, k, num_sms);
  if (p.splits <= 1) return 0;
  const size_t items = static_cast<size_t>(R) * p.splits * 2;
  return items * kH * kDvHalf * 4 + items * 2 * kH * 4;
}
}  // namespace dsa
