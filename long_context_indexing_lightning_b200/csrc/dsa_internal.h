// Internal (host-side) interfaces between the C ABI layer and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>
#include <numeric>

#include "dsa.h"

namespace dsa {

// Per-device facts and resources, set up once per device (dsa_api.cu).
int device_sm_count(int dev);
uint32_t* device_error_word(int dev);  // nullptr if the set-up failed

// Encode a 2-D row-major tensor map (inner dimension contiguous) with
// 128-byte swizzle, zero fill out of bounds.  Returns false on failure.
bool make_tmap_2d(CUtensorMap* map, const void* base, CUtensorMapDataType dt, int elem_bytes, uint64_t inner,
                  uint64_t rows, uint32_t box_inner, uint32_t box_rows);

struct IndexerArgs {
  int device;
  cudaStream_t stream;
  int B, n_q, s_max, H, D;
  int dtype;  // dsa_dtype_t of q_idx / k_idx
  const void* q_idx;
  const float* q_scale;
  const void* k_idx;
  const float* k_scale;
  const float* w;
  const int32_t* ctx_len;
  const int32_t* q_pos0;
  int t_off;  // added to q_pos0[b]: position of this call's query 0 within its sequence
  float* scores;
  int64_t ld;
  float idx_scale;
  uint32_t* err;
  // Optional (one-query schedule only, see indexer_hist_plan): each CTA also
  // writes the first 11-bit digit histograms of the (at most two) score rows
  // its run of key tiles covers, [cta][2][2048] (second row's zero if none).
  uint32_t* hist_parts = nullptr;
};

// Largest grid for which the indexer writes score histograms.
constexpr int kMaxHistCtas = 256;
// Bytes of the histogram handoff between the indexer and the top-k.
constexpr size_t kHistPartsBytes = static_cast<size_t>(kMaxHistCtas) * 2 * 2048 * 4;
// CTAs of the indexer's one-query (decode) schedule on num_sms SMs.  The
// e4m3 instance is paced by its epilogue and takes every SM; the bf16 one is
// bound by HBM, which 7/8 of the SMs already saturate (128K decode, 148 SMs:
// 167 us at 128-132 CTAs against 177 us at 148, where the extra CTAs' loads
// only queue).
int indexer_decode_grid(int num_sms, bool fp8);
// Whether the indexer's one-query schedule for (B, n_q, s_max) on num_sms SMs
// can emit score histograms (every CTA's run spans at most two rows); if so,
// the run length (tiles per CTA) and the key tiles per row.
bool indexer_hist_plan(int B, int n_q, int s_max, int num_sms, bool fp8, int* per_cta, int* tpr);

struct TopkArgs {
  int device;
  cudaStream_t stream;
  int B, n_q, s_max, k;
  const float* scores;
  int64_t ld;
  const int32_t* ctx_len;
  const int32_t* q_pos0;
  int t_off;
  int32_t* idx;
  void* ws;
  size_t ws_bytes;
  uint32_t* err;
  // Optional: output index = remap[row * remap_ld + s] instead of s (a
  // selection among a candidate list whose entries are ascending indices).
  const int32_t* remap = nullptr;
  int64_t remap_ld = 0;
  // Optional: the indexer's partial first-digit histograms (IndexerArgs::
  // hist_parts, written with runs of hist_per_cta tiles, hist_tpr tiles a
  // row), summed per row instead of reading the row for them.
  const uint32_t* hist_parts = nullptr;
  int hist_per_cta = 0, hist_tpr = 0;
};

// Cache append (csrc/cache_append.cu): token (b, i) -> cache row pos[b] + i.
struct AppendArgs {
  const void* k_new;   // [B][n_new][idx_dim]
  const void* kv_new;  // [B][n_new] rows of kv_row_bytes
  const void* v_new;   // [B][n_new] rows of v_row_bytes, or null
  const int32_t* pos;  // [B]
  void* k_cache;       // [B][s_max] rows of k_row_bytes (E4M3: 128 codes)
  float* k_scale;      // [B][s_max] (E4M3 only)
  void* kv_cache;
  void* v_cache;
  int B, n_new, s_max;
  int64_t k_row_bytes, kv_row_bytes, v_row_bytes;
  uint32_t* err;
};
dsa_status_t cache_append(const AppendArgs& a, bool fp8, int k_new_dtype, cudaStream_t stream);

// Launch attribute for programmatic dependent launch (see pdl_wait()).
inline cudaLaunchAttribute pdl_attribute() {
  cudaLaunchAttribute a;
  a.id = cudaLaunchAttributeProgrammaticStreamSerialization;
  a.val.programmaticStreamSerializationAllowed = 1;
  return a;
}

struct AttnArgs {
  int device;
  cudaStream_t stream;
  int B, n_q, s_max, H, KVH, d_qk, d_v, k;
  int dtype;  // F32 or BF16
  const void* q;
  const void* kv;
  const void* v;
  const int32_t* idx;
  const int32_t* ctx_len;
  void* out;
  float* lse;
  float sm_scale;
  void* ws;
  size_t ws_bytes;
  uint32_t* err;
};

// Exact bf16 scores of listed candidate keys (csrc/indexer_rescore.cu).
struct RescoreArgs {
  int device;
  cudaStream_t stream;
  int B, n_q, s_max, H, D;
  int n_cand;               // entries listed per row (the first min(n_cand, pos + 1) are read)
  int t_off;
  const void* q_idx;        // [B][n_q][H][D] bf16
  const void* k_idx;        // [B][s_max][D] bf16
  const float* w;           // [B][n_q][H]
  const int32_t* cand;      // [B][n_q][cand_ld]
  int64_t cand_ld;
  const int32_t* ctx_len;
  const int32_t* q_pos0;
  float* out;               // [B][n_q][out_ld]
  int64_t out_ld;
  float idx_scale;
  uint32_t* err;
};
dsa_status_t indexer_rescore(const RescoreArgs& a);
bool indexer_rescore_supported(int H, int D);

// Y = X W^T on the tensor cores (csrc/proj_gemm.cu): X [M][K], W [N][K]
// bf16 row-major; columns [0, n_split) of Y go to out0 (bf16, row stride
// ld0), columns [n_split, N) to out1 (fp32, row stride ld1).
struct GemmArgs {
  int device;
  cudaStream_t stream;
  int M, N, K, n_split;
  const void* x;
  const void* w;
  void* out0;
  int64_t ld0;
  float* out1;
  int64_t ld1;
  uint32_t* err;
};
dsa_status_t proj_gemm(const GemmArgs& a);
bool proj_gemm_supported(int N, int K, int n_split);

dsa_status_t indexer_tc(const IndexerArgs& a);    // BF16 / E4M3, tensor cores
dsa_status_t indexer_simt(const IndexerArgs& a);  // F32, CUDA cores
bool indexer_tc_supported(int H, int D);

size_t topk_workspace_bytes(int B, int n_q, int s_max, int k);
dsa_status_t topk_radix(const TopkArgs& a);

size_t attn_workspace_bytes(int B, int n_q, int H, int d_qk, int d_v, int KVH, int k, int dtype);
dsa_status_t attn_tc(const AttnArgs& a);    // BF16 absorbed MLA, tensor cores
dsa_status_t attn_simt(const AttnArgs& a);  // F32 (and BF16 shapes the tensor path does not take)
bool attn_tc_supported(int H, int d_qk, int d_v, int KVH);
size_t attn_scratch_bytes(int B, int n_q, int k, int num_sms);

dsa_status_t selftest_wait_timeout(uint32_t* err, cudaStream_t stream);

dsa_status_t hadamard_quant(const void* x, int x_dtype, int64_t rows, int dim, uint8_t* x8, float* scale,
                            cudaStream_t stream);

}  // namespace dsa
