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
};

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
