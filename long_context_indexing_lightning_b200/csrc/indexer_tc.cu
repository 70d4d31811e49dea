// Lightning-indexer scores on the 5th-generation tensor cores.
//
// DeepSeek-V3.2 model doc (Transformers), section "DeepSeek Sparse Attention
// (DSA)", item 1: an index score of each query against all previous keys of
// the indexer's single-head key cache (width index_head_dim = 128), combined
// over index_n_heads = 64 heads.  Per (query t, key s):
//     I[t,s] = sum_h w[t,h] * ReLU(scale * <q[t,h,:], k[s,:]>)   (s <= pos(t))
// The FP8 instance (same item: the reference indexer runs in FP8 after a
// Hadamard rotation) multiplies the e4m3 codes and folds the per-row scales
// into the epilogue: I = k_scale[s] * sum_h (w * q_scale)[t,h] * ReLU(dot).
//
// Design (sm_100a):
//   * One tile = 128 keys (MMA M) x N = QG queries * H_I heads (MMA N), K = 128.
//     Keys on M means each epilogue thread owns one key's TMEM lane and does
//     the ReLU-weighted head reduction from its own registers.
//   * Warp-specialised persistent CTA: warp 0 issues TMA loads of key tiles
//     (a ring of shared-memory stages) and of the query block, warp 1 issues
//     tcgen05.mma into a ring of TMEM accumulators, the remaining warps run
//     the epilogue (tcgen05.ld, ReLU, weighted head sum, causal mask, store).
//   * Decode (one query per sequence) is HBM-bound on the key cache, so each
//     CTA takes a contiguous run of key tiles (query block loaded once per
//     sequence it touches).  Prefill is tensor-bound; its units are chunks of
//     key tiles handed out in a scrambled order so the causal triangle
//     balances across CTAs.  Key tiles wholly above the diagonal of a query
//     block are not computed; the epilogue only writes -inf there.
//   * Every mbarrier wait is bounded; on expiry the kernel records a timeout
//     in the error word, drains its copies and MMAs, frees TMEM and returns.
#include "dsa_common.cuh"
#include "dsa_internal.h"

namespace dsa {
namespace {

constexpr int kTileKeys = 128;  // MMA M
constexpr int kIdxDim = 128;    // D_I
constexpr int kHistBins = 2048; // first 11-bit digit of the order-preserving score key

template <bool kFP8, int kQG, int kHI, int kEpiWarps, int kStages, int kQBufs, bool kHist>
struct IdxCfg {
  static constexpr int N = kQG * kHI;
  static constexpr int kElem = kFP8 ? 1 : 2;
  static constexpr int kRowBytes = kIdxDim * kElem;          // 256 (bf16) or 128 (fp8)
  static constexpr int kKBlocks = kRowBytes / 128;           // 128-byte swizzle atoms along K
  static constexpr int kKTile = kTileKeys * kRowBytes;       // bytes of one key tile
  static constexpr int kQTile = N * kRowBytes;               // bytes of one query block
  static constexpr int kNumMma = kRowBytes / 32;             // each MMA consumes 32 bytes of K
  // one query a tile with 12 epilogue warps: three groups, two accumulators each
  static constexpr int kNumAcc = (kQG == 1 && kEpiWarps == 12) ? 6 : (N <= 64) ? 4 : (512 / N);  // TMEM accumulators
  static constexpr int kTmemCols = (kNumAcc * N <= 256) ? 256 : 512;
  static constexpr int kThreads = 64 + 32 * kEpiWarps;
  static constexpr int kEpiThreads = 32 * kEpiWarps;
  // shared memory offsets (from a 1024-aligned base)
  static constexpr int kOffK = 0;
  static constexpr int kOffQ = kOffK + kStages * kKTile;
  static constexpr int kOffW = kOffQ + kQBufs * kQTile;
  static constexpr int kOffBar = kOffW + 2 * kQG * kHI * 4;  // two weight buffers
  static constexpr int kNumBars = 2 * kStages + 2 * kQBufs + 2 * kNumAcc + 1;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  // first-digit histograms of the (at most two) score rows the CTA writes
  static constexpr int kOffHist = kOffMisc + 16;
  static constexpr int kHistWords = kHist ? 2 * kHistBins : 0;
  static constexpr int kSmemBytes = kOffHist + kHistWords * 4 + 1024;  // + alignment slack
  static_assert(!kHist || kQG == 1, "score histograms are built in the one-query (decode) schedule");
  static_assert(N % 16 == 0 && N >= 16 && N <= 256, "MMA N");
  static_assert(kHI % 16 == 0, "heads per query");
  // Epilogue warps in groups of four (one warp per TMEM lane quarter): with
  // one query a tile the groups take turns by key tile (8 warps: alternate
  // tiles; 12: every third), else they split the query block (8: two groups
  // of kQG / 2 queries; 16: four groups of kQG / 4)
  static constexpr bool kAltTiles = (kEpiWarps >= 8 && kQG == 1);
  static constexpr int kGroups = kAltTiles ? kEpiWarps / 4 : 1;
  static constexpr int kAccArrivals = kAltTiles ? 128 : kEpiThreads;
  // the query's head weights: in registers (one query a tile, up to 8
  // epilogue warps), else in shared memory
  static constexpr bool kWRegs = (kQG == 1 && kEpiWarps <= 8);
  static_assert(kEpiWarps == 4 || (kEpiWarps == 8 && (kQG % 2 == 0 || kQG == 1)) || (kEpiWarps == 12 && kQG == 1) ||
                    (kEpiWarps == 16 && kQG % 4 == 0),
                "epilogue split");
  static_assert(!kAltTiles || kNumAcc % kGroups == 0, "every group needs the same accumulators");
  static_assert(kNumAcc * N <= 512, "tensor memory");
  static_assert(kKTile % 1024 == 0 && kQTile % 1024 == 0, "swizzle atom alignment");
};

struct Unit {
  int b, t0, nq, L, p0, kt0, kt_comp, kt_end;
};

struct Sched {
  int B, n_q, s_max, G, tpr;  // tpr: key tiles per sequence row
  int contiguous;             // 1: each CTA walks one contiguous run of tiles
  int per_cta;                // contiguous: tiles per CTA
  int TPC, NC, nunits, scramble;  // scrambled: units of TPC tiles
  int t_off;                  // position offset of query 0 of this call within its sequence
};

// Walks the work of one CTA as units (one query block, a run of key tiles).
// Contiguous mode cuts the CTA's run of tiles at query-block boundaries (one
// division per unit); scrambled mode visits chunks of TPC tiles in a
// multiplicative-hash order.  Every role of the CTA walks the same sequence.
struct UnitIter {
  int i, end;
};

__device__ __forceinline__ UnitIter iter_begin(const Sched& S, int cta) {
  UnitIter it;
  if (S.contiguous) {
    const int64_t total = static_cast<int64_t>(S.B) * S.G * S.tpr;
    const int64_t beg = static_cast<int64_t>(cta) * S.per_cta;
    const int64_t end = beg + S.per_cta;
    it.i = static_cast<int>(beg < total ? beg : total);
    it.end = static_cast<int>(end < total ? end : total);
  } else {
    it.i = 0;
    it.end = (S.nunits - cta + static_cast<int>(gridDim.x) - 1) / static_cast<int>(gridDim.x);
  }
  return it;
}

template <int kQG>
__device__ __forceinline__ bool iter_next(const Sched& S, UnitIter& it, int cta, Unit& r,
                                          const int32_t* __restrict__ ctx_len, const int32_t* __restrict__ q_pos0) {
  if (it.i >= it.end) return false;
  int bg, ka, kb;
  if (S.contiguous) {
    bg = it.i / S.tpr;
    ka = it.i - bg * S.tpr;
    kb = min(S.tpr, ka + (it.end - it.i));
    it.i += kb - ka;
  } else {
    const int v = cta + it.i * static_cast<int>(gridDim.x);
    const int u = static_cast<int>((static_cast<int64_t>(v) * S.scramble) % S.nunits);
    ++it.i;
    const int c = u % S.NC;
    bg = u / S.NC;
    ka = c * S.TPC;
    kb = min(S.tpr, ka + S.TPC);
  }
  const int g = bg % S.G;
  r.b = bg / S.G;
  r.L = min(max(__ldg(ctx_len + r.b), 0), S.s_max);
  r.p0 = max(__ldg(q_pos0 + r.b), 0) + S.t_off;
  r.t0 = g * kQG;
  r.nq = min(kQG, S.n_q - r.t0);
  const int pmax = min(r.p0 + r.t0 + r.nq - 1, r.L - 1);
  const int ntiles = (r.L + kTileKeys - 1) / kTileKeys;
  r.kt0 = ka;
  r.kt_end = min(kb, ntiles);
  r.kt_comp = min(r.kt_end, pmax >= 0 ? pmax / kTileKeys + 1 : 0);
  if (r.kt_comp < r.kt0) r.kt_comp = r.kt0;
  return true;
}

template <bool kFP8, int kQG, int kHI, int kEpiWarps, int kStages, int kQBufs, bool kHist>
__global__ void __launch_bounds__(IdxCfg<kFP8, kQG, kHI, kEpiWarps, kStages, kQBufs, kHist>::kThreads, 1)
    indexer_tc_kernel(const __grid_constant__ CUtensorMap tmap_k, const __grid_constant__ CUtensorMap tmap_q,
                      const float* __restrict__ w, const float* __restrict__ q_scale,
                      const float* __restrict__ k_scale, const int32_t* __restrict__ ctx_len,
                      const int32_t* __restrict__ q_pos0, float* __restrict__ scores, int64_t ld,
                      float idx_scale, Sched S, uint32_t* err, uint32_t* __restrict__ hist_out) {
  using C = IdxCfg<kFP8, kQG, kHI, kEpiWarps, kStages, kQBufs, kHist>;
  pdl_wait();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_addr(smem);
  float* w_s = reinterpret_cast<float*>(smem + C::kOffW);
  const uint32_t bar0 = sbase + C::kOffBar;
  auto k_full = [&](int i) { return bar0 + 8u * i; };
  auto k_empty = [&](int i) { return bar0 + 8u * (kStages + i); };
  auto q_full = [&](int i) { return bar0 + 8u * (2 * kStages + i); };
  auto q_empty = [&](int i) { return bar0 + 8u * (2 * kStages + kQBufs + i); };
  auto acc_full = [&](int i) { return bar0 + 8u * (2 * kStages + 2 * kQBufs + i); };
  auto acc_empty = [&](int i) { return bar0 + 8u * (2 * kStages + 2 * kQBufs + C::kNumAcc + i); };
  const uint32_t mma_done = bar0 + 8u * (C::kNumBars - 1);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = lane_id();

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) { mbar_init(k_full(i), 1); mbar_init(k_empty(i), 1); }
    for (int i = 0; i < kQBufs; ++i) { mbar_init(q_full(i), 1); mbar_init(q_empty(i), 1); }
    for (int i = 0; i < C::kNumAcc; ++i) { mbar_init(acc_full(i), 1); mbar_init(acc_empty(i), C::kAccArrivals); }
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  uint32_t* hist_s = reinterpret_cast<uint32_t*>(smem + C::kOffHist);
  if constexpr (kHist) {
    for (int i = threadIdx.x; i < C::kHistWords; i += C::kThreads) hist_s[i] = 0u;
  }
  if (warp == 1) {
    tmem_alloc(smem_addr(tmem_slot), C::kTmemCols);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_map(&tmap_k);
    tma_prefetch_map(&tmap_q);
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem_base = *tmem_slot;

  const int cta = blockIdx.x;

  if (warp == 0) {
    // ------------------------------------------------ TMA producer --
    if (lane == 0) {
      int st = 0, qb = 0;
      uint32_t kph = 0, qph = 0;
      int last_bg = -1;
      const uint64_t key_policy = l2_evict_first();
      uint32_t issued_k[kStages];
      uint32_t issued_q[kQBufs];
      for (int i = 0; i < kStages; ++i) issued_k[i] = 0;
      for (int i = 0; i < kQBufs; ++i) issued_q[i] = 0;
      UnitIter it = iter_begin(S, cta);
      Unit U;
      while (iter_next<kQG>(S, it, cta, U, ctx_len, q_pos0)) {
        if (U.kt_comp <= U.kt0) continue;
        const int bg = U.b * S.G + U.t0 / kQG;
        if (bg != last_bg) {
          if (last_bg >= 0) { if (++qb == kQBufs) { qb = 0; qph ^= 1; } }
          if (!mbar_wait(q_empty(qb), qph ^ 1, abort_flag, err)) break;
          mbar_arrive_expect_tx(q_full(qb), C::kQTile);
          const int qrow = (U.b * S.n_q + U.t0) * kHI;
          const uint32_t qdst = sbase + C::kOffQ + qb * C::kQTile;
#pragma unroll
          for (int kb = 0; kb < C::kKBlocks; ++kb)
            tma_load_2d(qdst + kb * C::N * 128, &tmap_q, q_full(qb), kb * (128 / C::kElem), qrow);
          issued_q[qb]++;
          last_bg = bg;
        }
        bool ok = true;
        for (int kt = U.kt0; kt < U.kt_comp; ++kt) {
          if (!mbar_wait(k_empty(st), kph ^ 1, abort_flag, err)) { ok = false; break; }
          mbar_arrive_expect_tx(k_full(st), C::kKTile);
          const int krow = U.b * S.s_max + kt * kTileKeys;
          const uint32_t kdst = sbase + C::kOffK + st * C::kKTile;
          // decode reads each key tile once: marked first to leave L2, so the
          // score rows (read next by the top-k) stay there; prefill re-reads
          // key tiles across query blocks and keeps the default
#pragma unroll
          for (int kb = 0; kb < C::kKBlocks; ++kb) {
            if constexpr (kQG == 1)
              tma_load_2d_hint(kdst + kb * kTileKeys * 128, &tmap_k, k_full(st), kb * (128 / C::kElem), krow,
                               key_policy);
            else
              tma_load_2d(kdst + kb * kTileKeys * 128, &tmap_k, k_full(st), kb * (128 / C::kElem), krow);
          }
          issued_k[st]++;
          if (++st == kStages) { st = 0; kph ^= 1; }
        }
        if (!ok) break;
      }
      // Drain: every copy this thread issued has landed before the CTA exits.
      volatile int never = 0;
      for (int i = 0; i < kStages; ++i)
        if (issued_k[i]) mbar_wait(k_full(i), (issued_k[i] - 1) & 1, &never, err);
      for (int i = 0; i < kQBufs; ++i)
        if (issued_q[i]) mbar_wait(q_full(i), (issued_q[i] - 1) & 1, &never, err);
    }
  } else if (warp == 1) {
    // ------------------------------------------------- MMA issuer --
    if (lane == 0) {
      constexpr uint32_t idesc = kFP8 ? idesc_e4m3_f32(kTileKeys, C::N) : idesc_bf16_f32(kTileKeys, C::N);
      const uint64_t a_desc0 = sdesc_kmajor_sw128(sbase + C::kOffK);
      int st = 0, qb = 0, ab = 0;
      uint32_t kph = 0, qph = 0, aph = 0;
      int last_bg = -1;
      UnitIter it = iter_begin(S, cta);
      Unit U;
      while (iter_next<kQG>(S, it, cta, U, ctx_len, q_pos0)) {
        if (U.kt_comp <= U.kt0) continue;
        const int bg = U.b * S.G + U.t0 / kQG;
        if (bg != last_bg) {
          if (last_bg >= 0) {
            tc_commit(q_empty(qb));
            if (++qb == kQBufs) { qb = 0; qph ^= 1; }
          }
          if (!mbar_wait(q_full(qb), qph, abort_flag, err)) break;
          last_bg = bg;
        }
        const uint64_t bd0 = sdesc_kmajor_sw128(sbase + C::kOffQ + qb * C::kQTile);
        bool ok = true;
        for (int kt = U.kt0; kt < U.kt_comp; ++kt) {
          if (!mbar_wait(acc_empty(ab), aph ^ 1, abort_flag, err)) { ok = false; break; }
          if (!mbar_wait(k_full(st), kph, abort_flag, err)) { ok = false; break; }
          tc_fence_after_sync();
          const uint32_t d = tmem_base + static_cast<uint32_t>(ab * C::N);
          const uint64_t ad0 = a_desc0 + static_cast<uint64_t>((st * C::kKTile) >> 4);
#pragma unroll
          for (int kk = 0; kk < C::kNumMma; ++kk) {
            // descriptor start addresses advance in 16-byte units
            const uint32_t a_off = ((kk * 32) / 128) * kTileKeys * 128 + (kk * 32) % 128;
            const uint32_t b_off = ((kk * 32) / 128) * C::N * 128 + (kk * 32) % 128;
            if (kFP8) tc_mma_f8(d, ad0 + (a_off >> 4), bd0 + (b_off >> 4), idesc, kk > 0 ? 1u : 0u);
            else tc_mma_f16(d, ad0 + (a_off >> 4), bd0 + (b_off >> 4), idesc, kk > 0 ? 1u : 0u);
          }
          tc_commit(k_empty(st));
          tc_commit(acc_full(ab));
          if (++st == kStages) { st = 0; kph ^= 1; }
          if (++ab == C::kNumAcc) { ab = 0; aph ^= 1; }
        }
        if (!ok) break;
      }
      // All MMAs issued above are complete before TMEM is released.
      tc_commit(mma_done);
      volatile int never = 0;
      mbar_wait(mma_done, 0, &never, err);
    }
  } else {
    // --------------------------------------------------- epilogue --
    const int e = warp - 2;
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;  // key within the tile == TMEM lane
    const int grp = e >> 2;  // warp group
    // (a query block split over the groups: kQG / (kEpiWarps / 4) queries each)
    constexpr int kQPer = (kEpiWarps >= 8 && !C::kAltTiles) ? kQG / (kEpiWarps / 4) : kQG;
    const int jbeg = (kEpiWarps >= 8 && !C::kAltTiles) ? grp * kQPer : 0;
    const int jend = jbeg + kQPer;
    // alternate tiles: group g takes the CTA's computed tiles n = g, g + G, ...
    // for G groups (accumulator n % kNumAcc, phase (n / kNumAcc) & 1)
    constexpr int kStep = C::kAltTiles ? C::kGroups : 1;
    int ncomp = 0;  // tiles the CTA computed in earlier units
    const int tid_e = threadIdx.x - 64;
    int ab = C::kAltTiles ? grp : 0, wb = 0;
    uint32_t aph = 0;
    int last_bg = -1;
    float wreg[C::kWRegs ? kHI : 1];
    UnitIter it = iter_begin(S, cta);
    // histogram slot of a score row: 0 for the first row of this CTA's run, 1 for the next
    const int first_bg = S.tpr > 0 ? it.i / S.tpr : 0;
    Unit U;
    while (iter_next<kQG>(S, it, cta, U, ctx_len, q_pos0)) {
      if (U.kt_end <= U.kt0) continue;
      uint32_t* hslot = hist_s + ((U.b * S.G + U.t0 / kQG) == first_bg ? 0 : kHistBins);
      if (C::kWRegs && U.kt_comp > U.kt0) {
        // one query: its head weights live in registers
        const int bg = U.b * S.G + U.t0;
        if (bg != last_bg) {
          const int64_t o = (static_cast<int64_t>(U.b) * S.n_q + U.t0) * kHI;
#pragma unroll
          for (int h = 0; h < kHI; ++h) {
            float v = __ldg(w + o + h) * idx_scale;
            if (kFP8) v *= __ldg(q_scale + o + h);
            wreg[h] = v;
          }
          last_bg = bg;
        }
      } else if (U.kt_comp > U.kt0) {
        const int bg = U.b * S.G + U.t0 / kQG;
        if (bg != last_bg) {
          // head weights of this query block, with the score scale (and the
          // per-(query, head) FP8 scale) folded in; double-buffered so the
          // barrier only has to order writers against the previous readers
          wb ^= 1;
          named_bar_sync(1, C::kEpiThreads);
          float* wd = w_s + wb * kQG * kHI;
          for (int k = tid_e; k < kQG * kHI; k += C::kEpiThreads) {
            const int j = k / kHI, h = k % kHI;
            float v = 0.f;
            if (j < U.nq) {
              const int64_t o = (static_cast<int64_t>(U.b) * S.n_q + U.t0 + j) * kHI + h;
              v = __ldg(w + o) * idx_scale;
              if (kFP8) v *= __ldg(q_scale + o);
            }
            wd[k] = v;
          }
          named_bar_sync(1, C::kEpiThreads);
          last_bg = bg;
        }
      }
      const float* wd = w_s + wb * kQG * kHI;
      // FP8 key scales run four tiles ahead of the accumulators: a scale
      // loaded after the accumulator wait would put one DRAM latency on
      // every tile's critical path.
      const float* ks_row = kFP8 ? k_scale + static_cast<int64_t>(U.b) * S.s_max + row : nullptr;
      auto load_ks = [&](int t) -> float {
        return (t < U.kt_comp && t * kTileKeys + row < U.L) ? __ldg(ks_row + t * kTileKeys) : 1.f;
      };
      const int kt_first = C::kAltTiles ? U.kt0 + (((grp - ncomp) % kStep) + kStep) % kStep : U.kt0;
      if (C::kAltTiles && U.kt_comp > U.kt0) ncomp += U.kt_comp - U.kt0;
      // One key tile of the epilogue (FP8: its keys' scale ks); false if a
      // wait expired.
      auto tile = [&](int kt, float ks) -> bool {
        if (!mbar_wait_warp(acc_full(ab), aph, abort_flag, err)) return false;
        tc_fence_after_sync();
        const int s = kt * kTileKeys + row;
        const uint32_t tl = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + static_cast<uint32_t>(ab * C::N);
        if constexpr (kQG == 1 && kHI == 64) {
          float v0[32], v1[32];
          tmem_ld32x2(tl, tl + 32, v0, v1);
          float acc0 = 0.f, acc1 = 0.f, acc2 = 0.f, acc3 = 0.f;
#pragma unroll
          for (int x = 0; x < 32; x += 2) {
            // (weights from shared memory: every lane reads the same word)
            const float w0 = C::kWRegs ? wreg[x] : wd[x], w1 = C::kWRegs ? wreg[x + 1] : wd[x + 1];
            const float w2 = C::kWRegs ? wreg[32 + x] : wd[32 + x], w3 = C::kWRegs ? wreg[33 + x] : wd[33 + x];
            acc0 = fmaf(w0, fmaxf(v0[x], 0.f), acc0);
            acc1 = fmaf(w1, fmaxf(v0[x + 1], 0.f), acc1);
            acc2 = fmaf(w2, fmaxf(v1[x], 0.f), acc2);
            acc3 = fmaf(w3, fmaxf(v1[x + 1], 0.f), acc3);
          }
          if (s < U.L) {
            const int p = U.p0 + U.t0;
            const float v = ((acc0 + acc1) + (acc2 + acc3)) * ks;
            scores[(static_cast<int64_t>(U.b) * S.n_q + U.t0) * ld + s] = (s <= p) ? v : -INFINITY;
            if constexpr (kHist) {
              if (s <= p) atomicAdd(&hslot[float_order_key(v) >> 21], 1u);
            }
          }
        } else
#pragma unroll 1
        for (int j = jbeg; j < jend; ++j) {
          float acc0 = 0.f, acc1 = 0.f;
          constexpr int kChunk = (kHI % 32 == 0) ? 32 : 16;
#pragma unroll
          for (int c = 0; c < kHI; c += kChunk) {
            float v[kChunk];
            if (kChunk == 32) tmem_ld32(tl + j * kHI + c, v);
            else tmem_ld16(tl + j * kHI + c, v);
#pragma unroll
            for (int x = 0; x < kChunk; x += 2) {
              acc0 = fmaf(wd[j * kHI + c + x], fmaxf(v[x], 0.f), acc0);
              acc1 = fmaf(wd[j * kHI + c + x + 1], fmaxf(v[x + 1], 0.f), acc1);
            }
          }
          if (j < U.nq && s < U.L) {
            const int p = U.p0 + U.t0 + j;
            const float v = (acc0 + acc1) * ks;
            scores[(static_cast<int64_t>(U.b) * S.n_q + U.t0 + j) * ld + s] = (s <= p) ? v : -INFINITY;
            if constexpr (kHist) {
              if (s <= p) atomicAdd(&hslot[float_order_key(v) >> 21], 1u);
            }
          }
        }
        tc_fence_before_sync();
        mbar_arrive(acc_empty(ab));
        ab += kStep;
        if (ab >= C::kNumAcc) { ab -= C::kNumAcc; aph ^= 1; }
        return true;
      };
      bool ok = true;
      if constexpr (kFP8) {
        // unrolled four ways so that each scale register is read four tiles
        // after its load, with no register moves in between (a move of a
        // load still in flight would wait for it)
        float ks0 = load_ks(kt_first), ks1 = load_ks(kt_first + kStep), ks2 = load_ks(kt_first + 2 * kStep),
              ks3 = load_ks(kt_first + 3 * kStep);
        for (int kt = kt_first; ok && kt < U.kt_comp; kt += 4 * kStep) {
          ok = tile(kt, ks0);
          ks0 = load_ks(kt + 4 * kStep);
          if (!ok || kt + kStep >= U.kt_comp) break;
          ok = tile(kt + kStep, ks1);
          ks1 = load_ks(kt + 5 * kStep);
          if (!ok || kt + 2 * kStep >= U.kt_comp) break;
          ok = tile(kt + 2 * kStep, ks2);
          ks2 = load_ks(kt + 6 * kStep);
          if (!ok || kt + 3 * kStep >= U.kt_comp) break;
          ok = tile(kt + 3 * kStep, ks3);
          ks3 = load_ks(kt + 7 * kStep);
        }
      } else {
        for (int kt = kt_first; ok && kt < U.kt_comp; kt += kStep) ok = tile(kt, 1.f);
      }
      if (!ok) break;
      // key tiles entirely after every query of the block: -inf only
      for (int kt = U.kt_comp + (C::kAltTiles ? grp : 0); kt < U.kt_end; kt += kStep) {
        const int s = kt * kTileKeys + row;
        if (s < U.L)
          for (int j = jbeg; j < min(jend, U.nq); ++j)
            scores[(static_cast<int64_t>(U.b) * S.n_q + U.t0 + j) * ld + s] = -INFINITY;
      }
    }
    if constexpr (kHist) {
      // this CTA's partial first-digit histograms of its first and second
      // score rows (zeros where it wrote none): the top-k sums them
      named_bar_sync(2, C::kEpiThreads);
      uint32_t* dst = hist_out + static_cast<int64_t>(cta) * C::kHistWords;
      for (int i = tid_e; i < C::kHistWords; i += C::kEpiThreads) dst[i] = hist_s[i];
    }
  }

  pdl_trigger();
  tc_fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after_sync();
    tmem_dealloc(tmem_base, C::kTmemCols);
  }
}

template <bool kFP8, int kQG, int kHI, int kEpiWarps, int kStages, int kQBufs, bool kHist>
dsa_status_t launch_indexer_tc(const IndexerArgs& a) {
  using C = IdxCfg<kFP8, kQG, kHI, kEpiWarps, kStages, kQBufs, kHist>;
  auto kern = indexer_tc_kernel<kFP8, kQG, kHI, kEpiWarps, kStages, kQBufs, kHist>;
  const int dev = a.device;
  const int num_sms = device_sm_count(dev);

  CUtensorMap tmk, tmq;
  const CUtensorMapDataType dt = kFP8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  const uint32_t box_inner = 128 / C::kElem;
  if (!make_tmap_2d(&tmk, a.k_idx, dt, C::kElem, kIdxDim, static_cast<uint64_t>(a.B) * a.s_max, box_inner,
                    kTileKeys))
    return DSA_ERR_CUDA;
  if (!make_tmap_2d(&tmq, a.q_idx, dt, C::kElem, kIdxDim, static_cast<uint64_t>(a.B) * a.n_q * kHI, box_inner,
                    C::N))
    return DSA_ERR_CUDA;

  Sched S;
  S.B = a.B;
  S.n_q = a.n_q;
  S.s_max = a.s_max;
  S.t_off = a.t_off;
  S.G = (a.n_q + kQG - 1) / kQG;
  S.tpr = (a.s_max + kTileKeys - 1) / kTileKeys;
  const int64_t total_tiles = static_cast<int64_t>(a.B) * S.G * S.tpr;
  if (total_tiles > INT32_MAX / 2) return DSA_ERR_UNSUPPORTED;
  const bool decode_like = (kQG == 1);
  S.contiguous = decode_like ? 1 : 0;
  S.TPC = decode_like ? 1 : std::min(16, S.tpr);
  S.NC = (S.tpr + S.TPC - 1) / S.TPC;
  S.nunits = static_cast<int>(static_cast<int64_t>(a.B) * S.G * S.NC);
  const int64_t work = decode_like ? total_tiles : S.nunits;
  const int grid = static_cast<int>(std::min<int64_t>(work, decode_like ? indexer_decode_grid(num_sms, kFP8) : num_sms));
  S.per_cta = static_cast<int>((total_tiles + grid - 1) / grid);
  // multiplier coprime to nunits for the scrambled order
  int64_t mult = 40503;
  while (std::gcd(mult, static_cast<int64_t>(S.nunits)) != 1) mult += 2;
  S.scramble = static_cast<int>(mult % S.nunits == 0 ? 1 : mult % S.nunits);

  static bool attr_done[64] = {};
  if (dev < 64 && !attr_done[dev]) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes) != cudaSuccess)
      return DSA_ERR_CUDA;
    attr_done[dev] = true;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid), 1, 1);
  cfg.blockDim = dim3(C::kThreads, 1, 1);
  cfg.dynamicSmemBytes = C::kSmemBytes;
  cfg.stream = a.stream;
  cudaLaunchAttribute attr[1] = {pdl_attribute()};
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, tmk, tmq, a.w, a.q_scale, a.k_scale, a.ctx_len, a.q_pos0,
                                           a.scores, a.ld, a.idx_scale, S, a.err, a.hist_parts);
  return e == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

}  // namespace

int indexer_decode_grid(int num_sms, bool fp8) { return fp8 ? num_sms : std::max(1, num_sms * 7 / 8); }

bool indexer_hist_plan(int B, int n_q, int s_max, int num_sms, bool fp8, int* per_cta, int* tpr) {
  // the decode schedule: one query per tile, each CTA a contiguous run of
  // key tiles; histograms only when a run spans at most two score rows
  if (n_q != 1 || B <= 0 || s_max <= 0 || num_sms <= 0 || num_sms > kMaxHistCtas) return false;
  const int64_t t = (s_max + kTileKeys - 1) / kTileKeys;
  const int64_t total = static_cast<int64_t>(B) * t;
  const int64_t grid = std::min<int64_t>(total, indexer_decode_grid(num_sms, fp8));
  const int64_t pc = (total + grid - 1) / grid;
  if (pc > t || total > INT32_MAX / 2) return false;
  *per_cta = static_cast<int>(pc);
  *tpr = static_cast<int>(t);
  return true;
}

dsa_status_t indexer_tc(const IndexerArgs& a) {
  // decode (n_q == 1): one query per tile; prefill: a block of queries filling N.
  const bool fp8 = (a.dtype == DSA_E4M3);
  if (a.D != kIdxDim) return DSA_ERR_UNSUPPORTED;
  const bool one = (a.n_q == 1);
  const bool hist = a.hist_parts != nullptr;
  if (hist) {
    int pc = 0, tp = 0;
    if (!indexer_hist_plan(a.B, a.n_q, a.s_max, device_sm_count(a.device), fp8, &pc, &tp)) return DSA_ERR_UNSUPPORTED;
  }
#define DSA_IDX_CASE(HI, QGP)                                                                  \
  if (a.H == HI) {                                                                             \
    if (one && hist) return fp8 ? launch_indexer_tc<true, 1, HI, ((HI) == 64 ? 12 : 8), 12, 2, true>(a) \
                                : launch_indexer_tc<false, 1, HI, 4, 5, 2, true>(a);           \
    if (one) return fp8 ? launch_indexer_tc<true, 1, HI, ((HI) == 64 ? 12 : 8), 12, 2, false>(a)        \
                        : launch_indexer_tc<false, 1, HI, 4, 5, 2, false>(a);                  \
    return fp8 ? launch_indexer_tc<true, QGP, HI, ((QGP) % 2 == 0 ? 8 : 4), 6, 1, false>(a)    \
               : launch_indexer_tc<false, QGP, HI, ((QGP) % 4 == 0 ? 16 : (QGP) % 2 == 0 ? 8 : 4), 4, 1, false>(a);  \
  }
  DSA_IDX_CASE(64, 4)
  DSA_IDX_CASE(32, 8)
  DSA_IDX_CASE(16, 16)
  DSA_IDX_CASE(128, 2)
#undef DSA_IDX_CASE
  return DSA_ERR_UNSUPPORTED;
}

}  // namespace dsa
