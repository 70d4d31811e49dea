// The indexer's projections, as one tensor-core GEMM.
//
// DeepSeek-V3.2 model doc (Transformers): the indexer scores queries taken
// from the low-rank query latent q_a_layernorm(q_a_proj(x)) through its
// `wq_b` projection, sized by q_lora_rank = 1536 (section "DeepSeek Sparse
// Attention (DSA)", the note on the query LoRA path), into index_n_heads =
// 64 heads of index_head_dim = 128 (section DeepseekV32Config); it keeps a
// single-head key of index_head_dim per token (the key-cache paragraph), and
// its head weights come from `weights_proj`, which the checkpoint keeps out
// of FP8 (section "Usage example").  Each is a plain linear map Y = X W^T:
//   wq_b:          X = q latent [T][1536]    W [8192][1536] -> q_idx [T][64][128] bf16
//   key + weights: X = hidden   [T][7168]    W [128 + 64][7168] -> k [T][128] bf16, w [T][64] fp32
// (the key projection and weights_proj read the same hidden state, so they
// run as one GEMM whose epilogue splits the output columns by type).
//
// Design (sm_100a): tiles of 128 rows x BN columns, K in 64-element steps
// (one 128-byte swizzle atom).  Persistent CTAs walk the tiles round robin;
// warp 0 streams X and W tiles with TMA into a ring of shared-memory stages,
// warp 1 issues tcgen05.mma (M = 128, N = BN, K = 16) into one of two TMEM
// accumulators, warps 2-5 drain an accumulator (tcgen05.ld, thread = row),
// convert and store while the next tile accumulates.  Every wait is bounded.
#include "dsa_common.cuh"
#include "dsa_internal.h"

namespace dsa {
namespace {

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}

constexpr int kBM = 128;   // rows per tile (MMA M)
constexpr int kBK = 64;    // K per stage: one 128-byte swizzle atom of bf16
constexpr int kEpiWarps = 4;
constexpr int kThreads = 64 + 32 * kEpiWarps;

template <int BN, int kStages>
struct GemmCfg {
  static constexpr int kATile = kBM * kBK * 2;       // 16 KB
  static constexpr int kBTile = BN * kBK * 2;
  static constexpr int kStage = kATile + kBTile;
  static constexpr int kOffBar = kStages * kStage;
  static constexpr int kNumBars = 2 * kStages + 4 + 1;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kSmemBytes = kOffMisc + 16 + 1024;
  static constexpr int kTmemCols = 2 * BN <= 256 ? 256 : 512;
  static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "MMA N");
  static_assert(kBTile % 1024 == 0 && kATile % 1024 == 0, "swizzle atom alignment");
  static_assert(kSmemBytes <= 232448, "shared memory");
};

struct GemmParams {
  int M, N, K;
  int n_split;        // columns [0, n_split) -> out0 (bf16), [n_split, N) -> out1 (fp32)
  __nv_bfloat16* out0;
  int64_t ld0;
  float* out1;
  int64_t ld1;
  int tiles_n, tiles;
  uint32_t* err;
};

template <int BN, int kStages>
__global__ void __launch_bounds__(kThreads, 1)
    proj_gemm_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_w,
                     GemmParams P) {
  using C = GemmCfg<BN, kStages>;
  pdl_wait();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_addr(smem);
  const uint32_t bar0 = sbase + C::kOffBar;
  auto full = [&](int i) { return bar0 + 8u * i; };
  auto empty = [&](int i) { return bar0 + 8u * (kStages + i); };
  auto acc_full = [&](int i) { return bar0 + 8u * (2 * kStages + i); };
  auto acc_empty = [&](int i) { return bar0 + 8u * (2 * kStages + 2 + i); };
  const uint32_t mma_done = bar0 + 8u * (2 * kStages + 4);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);
  const int warp = threadIdx.x >> 5, lane = lane_id();
  const int ksteps = P.K / kBK;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) { mbar_init(full(i), 1); mbar_init(empty(i), 1); }
    for (int i = 0; i < 2; ++i) { mbar_init(acc_full(i), 1); mbar_init(acc_empty(i), 32 * kEpiWarps); }
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_addr(tmem_slot), C::kTmemCols);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_map(&tmap_x);
    tma_prefetch_map(&tmap_w);
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------ TMA producer --
    if (lane == 0) {
      int st = 0;
      uint32_t ph = 0;
      uint32_t issued[kStages];
      for (int i = 0; i < kStages; ++i) issued[i] = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < P.tiles; tile += gridDim.x) {
        const int m0 = (tile / P.tiles_n) * kBM, n0 = (tile % P.tiles_n) * BN;
        for (int kb = 0; kb < ksteps; ++kb) {
          if (!mbar_wait(empty(st), ph ^ 1, abort_flag, P.err)) { ok = false; break; }
          mbar_arrive_expect_tx(full(st), C::kStage);
          const uint32_t dst = sbase + st * C::kStage;
          tma_load_2d(dst, &tmap_x, full(st), kb * kBK, m0);
          tma_load_2d(dst + C::kATile, &tmap_w, full(st), kb * kBK, n0);
          issued[st]++;
          if (++st == kStages) { st = 0; ph ^= 1; }
        }
      }
      volatile int never = 0;
      for (int i = 0; i < kStages; ++i)
        if (issued[i]) mbar_wait(full(i), (issued[i] - 1) & 1, &never, P.err);
    }
  } else if (warp == 1) {
    // -------------------------------------------------------- MMA issue --
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(kBM, BN);
      const uint64_t a0 = sdesc_kmajor_sw128(sbase);
      const uint64_t b0 = sdesc_kmajor_sw128(sbase + C::kATile);
      int st = 0, ab = 0;
      uint32_t ph = 0, aph = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < P.tiles; tile += gridDim.x) {
        if (!mbar_wait(acc_empty(ab), aph ^ 1, abort_flag, P.err)) break;
        tc_fence_after_sync();
        const uint32_t d = tmem + static_cast<uint32_t>(ab * BN);
        for (int kb = 0; kb < ksteps; ++kb) {
          if (!mbar_wait(full(st), ph, abort_flag, P.err)) { ok = false; break; }
          tc_fence_after_sync();
          const uint64_t so = static_cast<uint64_t>((st * C::kStage) >> 4);
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk)
            tc_mma_f16(d, a0 + so + ((kk * 32) >> 4), b0 + so + ((kk * 32) >> 4), idesc, (kb | kk) ? 1u : 0u);
          tc_commit(empty(st));
          if (++st == kStages) { st = 0; ph ^= 1; }
        }
        if (!ok) break;
        tc_commit(acc_full(ab));
        if (++ab == 2) { ab = 0; aph ^= 1; }
      }
      tc_commit(mma_done);
      volatile int never = 0;
      mbar_wait(mma_done, 0, &never, P.err);
    }
  } else {
    // --------------------------------------------------------- epilogue --
    const int quarter = warp & 3;
    const int row_in = quarter * 32 + lane;  // tile row == TMEM lane
    int ab = 0;
    uint32_t aph = 0;
    for (int tile = blockIdx.x; tile < P.tiles; tile += gridDim.x) {
      const int m0 = (tile / P.tiles_n) * kBM, n0 = (tile % P.tiles_n) * BN;
      if (!mbar_wait_warp(acc_full(ab), aph, abort_flag, P.err)) break;
      tc_fence_after_sync();
      const int m = m0 + row_in;
      const uint32_t tl = tmem + (static_cast<uint32_t>(quarter * 32) << 16) + static_cast<uint32_t>(ab * BN);
#pragma unroll 1
      for (int c = 0; c < BN; c += 32) {
        float v[32];
        tmem_ld32(tl + c, v);
        if (m >= P.M) continue;
        const int n = n0 + c;  // 32 columns, never straddling n_split (a multiple of 32)
        if (n < P.n_split) {
          __nv_bfloat16* dst = P.out0 + static_cast<int64_t>(m) * P.ld0 + n;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint4 u;
            u.x = pack_bf16x2(v[q * 8 + 0], v[q * 8 + 1]);
            u.y = pack_bf16x2(v[q * 8 + 2], v[q * 8 + 3]);
            u.z = pack_bf16x2(v[q * 8 + 4], v[q * 8 + 5]);
            u.w = pack_bf16x2(v[q * 8 + 6], v[q * 8 + 7]);
            *reinterpret_cast<uint4*>(dst + q * 8) = u;
          }
        } else {
          float* dst = P.out1 + static_cast<int64_t>(m) * P.ld1 + (n - P.n_split);
#pragma unroll
          for (int q = 0; q < 8; ++q)
            *reinterpret_cast<float4*>(dst + q * 4) = make_float4(v[q * 4], v[q * 4 + 1], v[q * 4 + 2], v[q * 4 + 3]);
        }
      }
      tc_fence_before_sync();
      mbar_arrive(acc_empty(ab));
      if (++ab == 2) { ab = 0; aph ^= 1; }
    }
  }

  pdl_trigger();
  tc_fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after_sync();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

template <int BN, int kStages>
dsa_status_t launch_gemm(const GemmArgs& a) {
  using C = GemmCfg<BN, kStages>;
  auto kern = proj_gemm_kernel<BN, kStages>;
  CUtensorMap tx, tw;
  if (!make_tmap_2d(&tx, a.x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.K, a.M, kBK, kBM)) return DSA_ERR_CUDA;
  if (!make_tmap_2d(&tw, a.w, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.K, a.N, kBK, BN)) return DSA_ERR_CUDA;
  GemmParams P;
  P.M = a.M;
  P.N = a.N;
  P.K = a.K;
  P.n_split = a.n_split;
  P.out0 = static_cast<__nv_bfloat16*>(a.out0);
  P.ld0 = a.ld0;
  P.out1 = a.out1;
  P.ld1 = a.ld1;
  P.tiles_n = a.N / BN;
  const int64_t tiles = static_cast<int64_t>((a.M + kBM - 1) / kBM) * P.tiles_n;
  if (tiles > INT32_MAX) return DSA_ERR_UNSUPPORTED;
  P.tiles = static_cast<int>(tiles);
  P.err = a.err;
  const int grid = static_cast<int>(std::min<int64_t>(tiles, std::max(1, device_sm_count(a.device))));
  static bool attr_done[64] = {};
  if (a.device < 0 || a.device >= 64) return DSA_ERR_UNSUPPORTED;
  if (!attr_done[a.device]) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes) != cudaSuccess)
      return DSA_ERR_CUDA;
    attr_done[a.device] = true;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid), 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = C::kSmemBytes;
  cfg.stream = a.stream;
  cudaLaunchAttribute attr[1] = {pdl_attribute()};
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, tx, tw, P) == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

}  // namespace

bool proj_gemm_supported(int N, int K, int n_split) {
  if (K <= 0 || K % kBK != 0 || n_split < 0 || n_split > N || n_split % 32 != 0) return false;
  return N == 192 || (N > 0 && N % 256 == 0) || N == 128 || N == 64;
}

dsa_status_t proj_gemm(const GemmArgs& a) {
  if (a.M == 0) return DSA_OK;
  if (!proj_gemm_supported(a.N, a.K, a.n_split)) return DSA_ERR_UNSUPPORTED;
  if (a.N == 192) return launch_gemm<192, 4>(a);
  if (a.N == 128) return launch_gemm<128, 6>(a);
  if (a.N == 64) return launch_gemm<64, 8>(a);
  return launch_gemm<256, 4>(a);
}

}  // namespace dsa
