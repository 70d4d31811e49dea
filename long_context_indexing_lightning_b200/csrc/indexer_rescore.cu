// Exact bf16 index scores of listed candidate keys, on the tensor cores.
//
// DeepSeek-V3.2 model doc (Transformers), section "DeepSeek Sparse Attention
// (DSA)", item 1: the reference indexer runs in FP8 after a Hadamard
// rotation, and FP8 is only a precision optimisation of the same score.  The
// e4m3 indexer here keeps the top (index_topk + margin) keys of its FP8
// scores; this kernel recomputes those candidates' scores from the bf16 key
// rows, exactly as the bf16 indexer scores them,
//     I[t,s] = sum_h w[t,h] * ReLU(scale * <q[t,h,:], k[s,:]>),
// and the final top-index_topk is taken over the recomputed scores.
//
// One tile = 128 candidates (MMA M, gathered key rows) x H_I heads (MMA N,
// the query's index-head block), K = 128.  Each CTA takes a run of tiles of
// one query row: its four warps gather the tile's 128 key rows (cp.async, 16
// bytes a lane, two rows a warp per instruction) into the 128-byte-swizzled
// K-major layout the MMA reads, double-buffered so the next tile's gather
// overlaps this tile's MMA and epilogue; thread 0 issues the MMAs into one of
// two TMEM accumulators; each thread then owns one candidate (its TMEM lane)
// and reduces its H_I head columns (ReLU, weight, sum) from its registers.
#include "dsa_common.cuh"
#include "dsa_internal.h"

namespace dsa {
namespace {

constexpr int kTileRows = 128;  // candidates per tile (MMA M)
constexpr int kDim = 128;       // D_I
constexpr int kThreads = 128;
constexpr int kAtom = kTileRows * 128;  // one 64-column atom of a tile: 16 KB

template <int kHI>
struct RsCfg {
  static constexpr int kKTile = 2 * kAtom;            // 32 KB of key rows
  static constexpr int kQAtom = kHI * 128;
  static constexpr int kQTile = 2 * kQAtom;           // the query block
  static constexpr int kOffK = 0;
  static constexpr int kOffQ = kOffK + 2 * kKTile;
  static constexpr int kOffW = kOffQ + kQTile;
  static constexpr int kOffBar = kOffW + kHI * 4;
  static constexpr int kOffMisc = kOffBar + 2 * 8;
  static constexpr int kSmemBytes = kOffMisc + 16 + 1024;
  static constexpr int kTmemCols = (2 * kHI <= 128) ? 128 : 256;
  static_assert(kQAtom % 1024 == 0, "swizzle atom alignment");
};

struct RsParams {
  const uint16_t* q;       // [R][H_I][128] bf16
  const uint16_t* k;       // [B][s_max][128] bf16
  const float* w;          // [R][H_I]
  const int32_t* cand;     // [R][cand_ld]: ascending key indices, -1 padding
  const int32_t* ctx_len;  // [B]
  const int32_t* q_pos0;   // [B]
  float* out;              // [R][out_ld]
  int64_t cand_ld, out_ld;
  int n_q, s_max, n_cand, t_off, tiles_per_cta, ctas_per_row;
  float idx_scale;
  uint32_t* err;
};

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}

template <int kHI>
__global__ void __launch_bounds__(kThreads, 1) indexer_rescore_kernel(RsParams P) {
  using C = RsCfg<kHI>;
  pdl_wait();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_addr(smem);
  float* w_s = reinterpret_cast<float*>(smem + C::kOffW);
  const uint32_t bar0 = sbase + C::kOffBar;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);
  const int tid = threadIdx.x, warp = tid >> 5, lane = lane_id();

  const int r = blockIdx.x / P.ctas_per_row;
  const int part = blockIdx.x % P.ctas_per_row;
  const int b = r / P.n_q, t = r % P.n_q;
  const int L = min(max(__ldg(P.ctx_len + b), 0), P.s_max);
  const int pos = __ldg(P.q_pos0 + b) + P.t_off + t;
  const int nvalid = max(0, min(P.n_cand, min(pos + 1, L)));  // listed candidates of this row
  const int ntiles = (nvalid + kTileRows - 1) / kTileRows;
  const int j0 = part * P.tiles_per_cta;
  const int j1 = min(ntiles, j0 + P.tiles_per_cta);
  if (j0 >= j1) {
    pdl_trigger();
    return;
  }
  const int32_t* cand = P.cand + static_cast<int64_t>(r) * P.cand_ld;
  const char* k_b = reinterpret_cast<const char*>(P.k) + static_cast<int64_t>(b) * P.s_max * kDim * 2;

  if (tid == 0) {
    mbar_init(bar0, 1);
    mbar_init(bar0 + 8, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_addr(tmem_slot), C::kTmemCols);
    tmem_relinquish();
  }
  if (tid < kHI) w_s[tid] = __ldg(P.w + static_cast<int64_t>(r) * kHI + tid) * P.idx_scale;
  // the query block: head rows, 16-byte chunk c of row h at chunk c ^ (h & 7)
  {
    const char* qb = reinterpret_cast<const char*>(P.q) + static_cast<int64_t>(r) * kHI * kDim * 2;
    for (int i = tid; i < kHI * 16; i += kThreads) {
      const int h = i >> 4, c = i & 15;
      const uint32_t dst = sbase + C::kOffQ + (c >> 3) * C::kQAtom + h * 128 + (((c & 7) ^ (h & 7)) << 4);
      cp_async16(dst, qb + h * kDim * 2 + c * 16, 16u);
    }
  }
  // gather of tile j into stage st: lane l of warp w moves chunk l % 16 of
  // tile row 8 i + 2 w + l / 16 for i = 0..15; rows past the list are zero
  bool bad = false;
  // (the sixteen list entries a lane needs are loaded first, all in flight
  // together, then the copies issued)
  auto gather = [&](int j, int st) {
    const int c = lane & 15;
    const uint32_t base = sbase + C::kOffK + st * C::kKTile + (c >> 3) * kAtom;
    int sv[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const int slot = j * kTileRows + i * 8 + warp * 2 + (lane >> 4);
      sv[i] = slot < nvalid ? __ldg(cand + slot) : -1;
    }
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const int row = i * 8 + warp * 2 + (lane >> 4);
      const int slot = j * kTileRows + row;
      int s = sv[i];
      if (slot < nvalid && (s < 0 || s >= L)) {  // a listed key outside the cache: zero row, flagged
        bad = true;
        s = -1;
      }
      const char* src = k_b + (s >= 0 ? static_cast<int64_t>(s) * kDim * 2 + c * 16 : 0);
      cp_async16(base + row * 128 + (((c & 7) ^ (row & 7)) << 4), src, s >= 0 ? 16u : 0u);
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  };
  gather(j0, 0);  // (one group with the query block)
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_slot;

  constexpr uint32_t idesc = idesc_bf16_f32(kTileRows, kHI);
  const uint64_t a_desc0 = sdesc_kmajor_sw128(sbase + C::kOffK);
  const uint64_t b_desc0 = sdesc_kmajor_sw128(sbase + C::kOffQ);
  float* out = P.out + static_cast<int64_t>(r) * P.out_ld;
  bool failed = false;
  for (int j = j0; j < j1; ++j) {
    const int st = (j - j0) & 1;
    if (j + 1 < j1) {
      gather(j + 1, st ^ 1);
      asm volatile("cp.async.wait_group 1;" ::: "memory");
    } else {
      asm volatile("cp.async.wait_group 0;" ::: "memory");
    }
    // this thread's copies of tile j have landed: hand the tile to the
    // tensor cores (generic-proxy writes -> async-proxy reads)
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t d = tmem + static_cast<uint32_t>(st * kHI);
    if (tid == 0) {
      const uint64_t ad = a_desc0 + static_cast<uint64_t>((st * C::kKTile) >> 4);
#pragma unroll
      for (int kk = 0; kk < kDim / 16; ++kk) {
        const uint32_t a_off = ((kk * 32) / 128) * kAtom + (kk * 32) % 128;
        const uint32_t b_off = ((kk * 32) / 128) * C::kQAtom + (kk * 32) % 128;
        tc_mma_f16(d, ad + (a_off >> 4), b_desc0 + (b_off >> 4), idesc, kk > 0 ? 1u : 0u);
      }
      tc_commit(bar0 + 8u * st);
    }
    failed = !mbar_wait_warp(bar0 + 8u * st, ((j - j0) >> 1) & 1, abort_flag, P.err);
    if (__syncthreads_or(failed)) break;
    tc_fence_after_sync();
    // epilogue: thread = candidate row = TMEM lane
    const int row = warp * 32 + lane;
    const uint32_t tl = d + (static_cast<uint32_t>(warp * 32) << 16);
    float acc0 = 0.f, acc1 = 0.f;
#pragma unroll
    for (int c0 = 0; c0 < kHI; c0 += (kHI >= 32 ? 32 : 16)) {
      constexpr int kCh = kHI >= 32 ? 32 : 16;
      float v[kCh];
      if constexpr (kCh == 32) tmem_ld32(tl + c0, v);
      else tmem_ld16(tl + c0, v);
#pragma unroll
      for (int x = 0; x < kCh; x += 2) {
        acc0 = fmaf(w_s[c0 + x], fmaxf(v[x], 0.f), acc0);
        acc1 = fmaf(w_s[c0 + x + 1], fmaxf(v[x + 1], 0.f), acc1);
      }
    }
    const int slot = j * kTileRows + row;
    if (slot < nvalid) out[slot] = acc0 + acc1;
    tc_fence_before_sync();
  }
  pdl_trigger();
  asm volatile("cp.async.wait_all;" ::: "memory");
  if (bad) raise_error(P.err, kErrBadIndex);
  tc_fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after_sync();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

template <int kHI>
dsa_status_t launch_rescore(const RescoreArgs& a) {
  using C = RsCfg<kHI>;
  auto kern = indexer_rescore_kernel<kHI>;
  const int64_t R = static_cast<int64_t>(a.B) * a.n_q;
  const int ntiles = (a.n_cand + kTileRows - 1) / kTileRows;
  if (R == 0 || ntiles == 0) return DSA_OK;
  const int num_sms = std::max(1, device_sm_count(a.device));
  // runs of tiles so that the grid covers about two CTAs per SM
  int64_t target = 2LL * num_sms;
  int parts = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(ntiles, (target + R - 1) / R)));
  const int tpc = (ntiles + parts - 1) / parts;
  parts = (ntiles + tpc - 1) / tpc;
  if (R * parts > INT32_MAX) return DSA_ERR_UNSUPPORTED;
  RsParams P;
  P.q = static_cast<const uint16_t*>(a.q_idx);
  P.k = static_cast<const uint16_t*>(a.k_idx);
  P.w = a.w;
  P.cand = a.cand;
  P.ctx_len = a.ctx_len;
  P.q_pos0 = a.q_pos0;
  P.out = a.out;
  P.cand_ld = a.cand_ld;
  P.out_ld = a.out_ld;
  P.n_q = a.n_q;
  P.s_max = a.s_max;
  P.n_cand = a.n_cand;
  P.t_off = a.t_off;
  P.tiles_per_cta = tpc;
  P.ctas_per_row = parts;
  P.idx_scale = a.idx_scale;
  P.err = a.err;
  static bool attr_done[64] = {};
  if (a.device < 0 || a.device >= 64) return DSA_ERR_UNSUPPORTED;
  if (!attr_done[a.device]) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes) != cudaSuccess)
      return DSA_ERR_CUDA;
    attr_done[a.device] = true;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(R * parts), 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = C::kSmemBytes;
  cfg.stream = a.stream;
  cudaLaunchAttribute attr[1] = {pdl_attribute()};
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, P) == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

}  // namespace

bool indexer_rescore_supported(int H, int D) { return D == kDim && (H == 16 || H == 32 || H == 64 || H == 128); }

dsa_status_t indexer_rescore(const RescoreArgs& a) {
  if (a.D != kDim) return DSA_ERR_UNSUPPORTED;
  switch (a.H) {
    case 16: return launch_rescore<16>(a);
    case 32: return launch_rescore<32>(a);
    case 64: return launch_rescore<64>(a);
    case 128: return launch_rescore<128>(a);
    default: return DSA_ERR_UNSUPPORTED;
  }
}

}  // namespace dsa
