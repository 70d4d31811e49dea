// C ABI of libdsa.so: argument checks, workspace layout, dispatch to the
// kernels, per-device set-up (SM count, error word, tensor-map encoder).
// The operations and their sources are documented in include/dsa.h.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <cmath>
#include <cstring>
#include <mutex>

#include "dsa.h"
#include "dsa_common.cuh"
#include "dsa_internal.h"

namespace dsa {

// Per-device error word: bit kErrTimeout / kErrBadIndex, set by kernels.
static __device__ uint32_t g_error_word[4];

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_mutex;
int g_sm_count[kMaxDevices] = {};
uint32_t* g_err_ptr[kMaxDevices] = {};
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

bool current_device(int* dev) { return cudaGetDevice(dev) == cudaSuccess && *dev >= 0 && *dev < kMaxDevices; }

// One-time set-up of `dev` (must be the current device): SM count and the
// device address of the error word.
bool ensure_device(int dev) {
  std::lock_guard<std::mutex> lock(g_mutex);
  if (g_sm_count[dev] > 0 && g_err_ptr[dev] != nullptr) return true;
  int sms = 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0) {
    (void)cudaGetLastError();  // consumed here, so it is not reported against a later call
    return false;
  }
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_error_word) != cudaSuccess || p == nullptr) {
    (void)cudaGetLastError();
    return false;
  }
  g_sm_count[dev] = sms;
  g_err_ptr[dev] = static_cast<uint32_t*>(p);
  return true;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

bool valid_dtype(int d) { return d == DSA_F32 || d == DSA_BF16 || d == DSA_E4M3; }

size_t elem_size(int dtype) { return dtype == DSA_F32 ? 4 : (dtype == DSA_BF16 ? 2 : 1); }

dsa_status_t check_shape(const dsa_shape_t* s) {
  if (s == nullptr) return DSA_ERR_INVALID_ARG;
  if (s->batch < 0 || s->n_q < 0 || s->s_max < 0) return DSA_ERR_INVALID_ARG;
  if (s->idx_heads <= 0 || s->idx_dim <= 0 || s->topk <= 0) return DSA_ERR_INVALID_ARG;
  if (s->heads <= 0 || s->d_qk <= 0 || s->d_v <= 0 || s->kv_heads <= 0) return DSA_ERR_INVALID_ARG;
  if (s->heads % s->kv_heads != 0) return DSA_ERR_INVALID_ARG;
  if (s->kv_heads == 1 && s->d_v > s->d_qk) return DSA_ERR_INVALID_ARG;
  if (!valid_dtype(s->idx_dtype) || !(s->attn_dtype == DSA_F32 || s->attn_dtype == DSA_BF16))
    return DSA_ERR_INVALID_ARG;
  if (!(s->idx_scale > 0.f) || !std::isfinite(s->idx_scale)) return DSA_ERR_INVALID_ARG;
  if (!std::isfinite(s->sm_scale)) return DSA_ERR_INVALID_ARG;
  if (s->q_chunk < 0 || s->idx_rescore < 0) return DSA_ERR_INVALID_ARG;
  if (static_cast<int64_t>(s->topk) + s->idx_rescore > INT32_MAX / 4) return DSA_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(s->batch) * s->s_max > INT32_MAX) return DSA_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(s->batch) * s->n_q * s->idx_heads > INT32_MAX) return DSA_ERR_UNSUPPORTED;
  return DSA_OK;
}

// ------------------------------------------------------------- stages --
dsa_status_t run_indexer(const dsa_shape_t* s, int dev, cudaStream_t st, int B, int n_q, int t_off,
                         const void* q_idx, const float* q_scale, const void* k_idx, const float* k_scale,
                         const float* w, const int32_t* ctx_len, const int32_t* q_pos0, float* scores,
                         int64_t ld, uint32_t* hist_parts = nullptr) {
  IndexerArgs a;
  a.hist_parts = hist_parts;
  a.device = dev;
  a.stream = st;
  a.B = B;
  a.n_q = n_q;
  a.s_max = s->s_max;
  a.H = s->idx_heads;
  a.D = s->idx_dim;
  a.dtype = s->idx_dtype;
  a.q_idx = q_idx;
  a.q_scale = q_scale;
  a.k_idx = k_idx;
  a.k_scale = k_scale;
  a.w = w;
  a.ctx_len = ctx_len;
  a.q_pos0 = q_pos0;
  a.t_off = t_off;
  a.scores = scores;
  a.ld = ld;
  a.idx_scale = s->idx_scale;
  a.err = g_err_ptr[dev];
  if (B == 0 || n_q == 0 || s->s_max == 0) return DSA_OK;
  if (s->idx_dtype == DSA_F32) return indexer_simt(a);
  return indexer_tc(a);
}

// Top-k of rows of `row_len` scores (the cache length, or the candidate list
// length when `remap` maps list slots to key indices).
dsa_status_t run_topk(int dev, cudaStream_t st, int B, int n_q, int t_off, int row_len, int k, const float* scores,
                      int64_t ld, const int32_t* ctx_len, const int32_t* q_pos0, int32_t* idx, void* ws,
                      size_t ws_bytes, const int32_t* remap = nullptr, int64_t remap_ld = 0,
                      const uint32_t* hist_parts = nullptr, int hist_per_cta = 0, int hist_tpr = 0) {
  TopkArgs a;
  a.hist_parts = hist_parts;
  a.hist_per_cta = hist_per_cta;
  a.hist_tpr = hist_tpr;
  a.device = dev;
  a.stream = st;
  a.B = B;
  a.n_q = n_q;
  a.s_max = row_len;
  a.k = k;
  a.remap = remap;
  a.remap_ld = remap_ld;
  a.scores = scores;
  a.ld = ld;
  a.ctx_len = ctx_len;
  a.q_pos0 = q_pos0;
  a.t_off = t_off;
  a.idx = idx;
  a.ws = ws;
  a.ws_bytes = ws_bytes;
  a.err = g_err_ptr[dev];
  if (B == 0 || n_q == 0) return DSA_OK;
  return topk_radix(a);
}

dsa_status_t run_rescore(const dsa_shape_t* s, int dev, cudaStream_t st, int B, int n_q, int t_off,
                         const void* q_idx, const void* k_idx, const float* w, const int32_t* cand, int64_t cand_ld,
                         int n_cand, const int32_t* ctx_len, const int32_t* q_pos0, float* out, int64_t out_ld) {
  RescoreArgs a;
  a.device = dev;
  a.stream = st;
  a.B = B;
  a.n_q = n_q;
  a.s_max = s->s_max;
  a.H = s->idx_heads;
  a.D = s->idx_dim;
  a.n_cand = n_cand;
  a.t_off = t_off;
  a.q_idx = q_idx;
  a.k_idx = k_idx;
  a.w = w;
  a.cand = cand;
  a.cand_ld = cand_ld;
  a.ctx_len = ctx_len;
  a.q_pos0 = q_pos0;
  a.out = out;
  a.out_ld = out_ld;
  a.idx_scale = s->idx_scale;
  a.err = g_err_ptr[dev];
  if (B == 0 || n_q == 0 || n_cand == 0) return DSA_OK;
  return indexer_rescore(a);
}

// The indexer -> top-k histogram handoff for a call over B x n_q queries:
// whether the indexer's schedule emits it (tensor-core indexer, one query per
// sequence, runs spanning at most two rows), and its run length and tiles per row.
struct HistPlan {
  bool on = false;
  int per_cta = 0, tpr = 0;
};
HistPlan hist_plan(const dsa_shape_t* s, int dev, int B, int n_q) {
  HistPlan h;
  if (s->idx_dtype == DSA_F32 || !indexer_tc_supported(s->idx_heads, s->idx_dim)) return h;
  h.on = indexer_hist_plan(B, n_q, s->s_max, device_sm_count(dev), s->idx_dtype == DSA_E4M3, &h.per_cta, &h.tpr);
  return h;
}

dsa_status_t run_attn(const dsa_shape_t* s, int dev, cudaStream_t st, int B, int n_q, const void* q, const void* kv,
                      const void* v, const int32_t* idx, const int32_t* ctx_len, void* out, float* lse, void* ws,
                      size_t ws_bytes) {
  AttnArgs a;
  a.device = dev;
  a.stream = st;
  a.B = B;
  a.n_q = n_q;
  a.s_max = s->s_max;
  a.H = s->heads;
  a.KVH = s->kv_heads;
  a.d_qk = s->d_qk;
  a.d_v = s->d_v;
  a.k = s->topk;
  a.dtype = s->attn_dtype;
  a.q = q;
  a.kv = kv;
  a.v = v;
  a.idx = idx;
  a.ctx_len = ctx_len;
  a.out = out;
  a.lse = lse;
  a.sm_scale = s->sm_scale;
  a.ws = ws;
  a.ws_bytes = ws_bytes;
  a.err = g_err_ptr[dev];
  if (B == 0 || n_q == 0) return DSA_OK;
  if (s->attn_dtype == DSA_BF16 && attn_tc_supported(a.H, a.d_qk, a.d_v, a.KVH)) return attn_tc(a);
  return attn_simt(a);
}

// Workspace layout of dsa_forward (all offsets 256-byte aligned).
struct FwdLayout {
  int chunk;          // queries per sequence per round
  int64_t ld;         // score row stride
  int kc;             // E4M3 with re-scoring: candidates per query (topk + idx_rescore), else 0
  size_t off_scores, off_idx, off_q8, off_qs, off_topk, off_attn, off_cand, off_rs, off_hist;
  size_t topk_bytes, attn_bytes;
  size_t total;
  // host-variant staging: two input slots (consecutive calls alternate, so a
  // call's inputs can be copied in while the previous call still reads its
  // own), offsets of each input within a slot, one output area
  size_t off_h_in[2];
  size_t off_h_qidx, off_h_w, off_h_q, off_h_ctx, off_h_pos;
  size_t off_h_out, off_h_lse;
  size_t total_host;
};

FwdLayout forward_layout(const dsa_shape_t* s) {
  FwdLayout L{};
  const int B = s->batch;
  L.chunk = (s->q_chunk > 0 && s->q_chunk < s->n_q) ? s->q_chunk : s->n_q;
  L.ld = static_cast<int64_t>(align_up(static_cast<size_t>(std::max(s->s_max, 1)), 4));
  size_t off = 0;
  L.off_scores = off;
  off = align_up(off + static_cast<size_t>(B) * L.chunk * L.ld * 4, 256);
  L.off_idx = off;
  off = align_up(off + static_cast<size_t>(B) * L.chunk * s->topk * 4, 256);
  L.off_q8 = off;
  L.off_qs = off;
  if (s->idx_dtype == DSA_E4M3) {
    off = align_up(off + static_cast<size_t>(B) * s->n_q * s->idx_heads * s->idx_dim, 256);
    L.off_qs = off;
    off = align_up(off + static_cast<size_t>(B) * s->n_q * s->idx_heads * 4, 256);
  }
  L.kc = (s->idx_dtype == DSA_E4M3 && s->idx_rescore > 0) ? s->topk + s->idx_rescore : 0;
  L.off_cand = off;
  off = align_up(off + static_cast<size_t>(B) * L.chunk * L.kc * 4, 256);
  L.off_rs = off;
  off = align_up(off + static_cast<size_t>(B) * L.chunk * L.kc * 4, 256);
  L.off_hist = off;
  if (L.chunk == 1) off = align_up(off + kHistPartsBytes, 256);
  L.off_topk = off;
  L.topk_bytes = topk_workspace_bytes(B, L.chunk, s->s_max, s->topk);
  off = align_up(off + L.topk_bytes, 256);
  L.off_attn = off;
  L.attn_bytes = attn_workspace_bytes(B, L.chunk, s->heads, s->d_qk, s->d_v, s->kv_heads, s->topk, s->attn_dtype);
  off = align_up(off + L.attn_bytes, 256);
  L.total = off;
  // staging for dsa_forward_host
  const size_t ai = elem_size(s->idx_dtype == DSA_E4M3 ? DSA_BF16 : s->idx_dtype);
  const size_t aa = elem_size(s->attn_dtype);
  size_t in = 0;
  L.off_h_qidx = in;
  in = align_up(in + static_cast<size_t>(B) * s->n_q * s->idx_heads * s->idx_dim * ai, 256);
  L.off_h_w = in;
  in = align_up(in + static_cast<size_t>(B) * s->n_q * s->idx_heads * 4, 256);
  L.off_h_q = in;
  in = align_up(in + static_cast<size_t>(B) * s->n_q * s->heads * s->d_qk * aa, 256);
  L.off_h_ctx = in;
  in = align_up(in + static_cast<size_t>(B) * 4, 256);
  L.off_h_pos = in;
  in = align_up(in + static_cast<size_t>(B) * 4, 256);
  L.off_h_in[0] = off;
  L.off_h_in[1] = off + in;
  off += 2 * in;
  L.off_h_out = off;
  off = align_up(off + static_cast<size_t>(B) * s->n_q * s->heads * s->d_v * aa, 256);
  L.off_h_lse = off;
  off = align_up(off + static_cast<size_t>(B) * s->n_q * s->heads * 4, 256);
  L.total_host = off;
  return L;
}

dsa_status_t check_indexer_inputs(const dsa_shape_t* s, const void* q_idx, const float* q_scale, const void* k_idx,
                                  const float* k_scale, const float* w, const int32_t* ctx_len,
                                  const int32_t* q_pos0) {
  if (!q_idx || !k_idx || !w || !ctx_len || !q_pos0) return DSA_ERR_INVALID_ARG;
  if (s->idx_dtype == DSA_E4M3 && (!q_scale || !k_scale)) return DSA_ERR_INVALID_ARG;
  if (s->idx_dtype != DSA_F32) {
    if (!aligned16(q_idx) || !aligned16(k_idx)) return DSA_ERR_INVALID_ARG;
    if (s->idx_dim != 128) return DSA_ERR_UNSUPPORTED;
    if (!indexer_tc_supported(s->idx_heads, s->idx_dim)) return DSA_ERR_UNSUPPORTED;
  } else {
    if (s->idx_dim > 256 || s->idx_heads > 128) return DSA_ERR_UNSUPPORTED;
  }
  return DSA_OK;
}

dsa_status_t check_attn_inputs(const dsa_shape_t* s, const void* q, const void* kv, const void* v, const void* idx,
                               const void* ctx_len, const void* out) {
  if (!q || !kv || !idx || !ctx_len || !out) return DSA_ERR_INVALID_ARG;
  if (s->kv_heads == 1 && v != nullptr) return DSA_ERR_INVALID_ARG;
  if (s->kv_heads > 1 && v == nullptr) return DSA_ERR_INVALID_ARG;
  if (s->attn_dtype == DSA_BF16 && attn_tc_supported(s->heads, s->d_qk, s->d_v, s->kv_heads)) {
    if (!aligned16(q) || !aligned16(kv) || !aligned16(out)) return DSA_ERR_INVALID_ARG;
    return DSA_OK;
  }
  const bool simt_ok = (s->d_qk == 32 && s->d_v == 32) || (s->d_qk == 64 && s->d_v == 64) ||
                       (s->d_qk == 128 && s->d_v == 128) || (s->d_qk == 576 && s->d_v == 512);
  return simt_ok ? DSA_OK : DSA_ERR_UNSUPPORTED;
}

}  // namespace

int device_sm_count(int dev) { return (dev >= 0 && dev < kMaxDevices) ? g_sm_count[dev] : 0; }

// The host-buffer entry points copy their inputs in on a stream of the
// library's own, into one of two staging slots of the workspace (consecutive
// calls alternate), so that a call's copies run while the previous call
// computes; the asynchronous one also copies the output back on a third
// stream, under the next call's indexer and top-k.  Created once per device
// on first use, with the events that join the streams:
//   g_ev_free[p]  the attention of the last call that used slot p is done
//                 (the next copy into slot p waits for it),
//   g_ev_in       the indexer inputs of a call are in its slot,
//   g_ev_q        the attention queries of a call are in its slot,
//   g_ev_attn     the attention of the last asynchronous call is done,
//   g_ev_out      the output copy of the last asynchronous call is done (the
//                 next call's attention, which rewrites the output, waits),
//   g_ev_join     the compute stream reached a call with a workspace other
//                 than the last one: the copy stream starts after it, since
//                 memory just handed out by a stream-ordered allocator may
//                 still be in use by earlier work on that stream.
cudaStream_t g_copy_stream[kMaxDevices] = {}, g_out_stream[kMaxDevices] = {};
cudaEvent_t g_ev_free[kMaxDevices][2] = {}, g_ev_in[kMaxDevices] = {}, g_ev_q[kMaxDevices] = {};
cudaEvent_t g_ev_attn[kMaxDevices] = {}, g_ev_out[kMaxDevices] = {}, g_ev_join[kMaxDevices] = {};
int g_slot[kMaxDevices] = {};
const void* g_last_ws[kMaxDevices] = {};
// Held by a host-buffer call from its slot choice to its last event record,
// so that calls from several host threads on one device cannot take the same
// staging slot or interleave their event records.
std::mutex g_host_mutex[kMaxDevices];
bool ensure_copy_stream(int dev) {
  std::lock_guard<std::mutex> lock(g_mutex);
  if (g_copy_stream[dev] != nullptr) return true;
  cudaStream_t s = nullptr, so = nullptr;
  cudaEvent_t ev[7] = {};
  if (cudaStreamCreateWithFlags(&s, cudaStreamNonBlocking) != cudaSuccess ||
      cudaStreamCreateWithFlags(&so, cudaStreamNonBlocking) != cudaSuccess)
    return false;
  for (cudaEvent_t& e : ev)
    if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) return false;
  g_ev_free[dev][0] = ev[0];
  g_ev_free[dev][1] = ev[1];
  g_ev_in[dev] = ev[2];
  g_ev_q[dev] = ev[3];
  g_ev_attn[dev] = ev[4];
  g_ev_out[dev] = ev[5];
  g_ev_join[dev] = ev[6];
  g_out_stream[dev] = so;
  g_copy_stream[dev] = s;
  return true;
}

uint32_t* device_error_word(int dev) { return (dev >= 0 && dev < kMaxDevices) ? g_err_ptr[dev] : nullptr; }

bool make_tmap_2d(CUtensorMap* map, const void* base, CUtensorMapDataType dt, int elem_bytes, uint64_t inner,
                  uint64_t rows, uint32_t box_inner, uint32_t box_rows) {
  {
    std::lock_guard<std::mutex> lock(g_mutex);
    if (g_encode == nullptr) {
      void* fn = nullptr;
      cudaDriverEntryPointQueryResult q;
      if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
          q != cudaDriverEntryPointSuccess || fn == nullptr)
        return false;
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
  }
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {inner * static_cast<uint64_t>(elem_bytes)};
  cuuint32_t box[2] = {box_inner, box_rows};
  cuuint32_t estr[2] = {1, 1};
  const CUresult r = g_encode(map, dt, 2, const_cast<void*>(base), dims, strides, box, estr,
                              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool indexer_tc_supported(int H, int D) { return D == 128 && (H == 16 || H == 32 || H == 64 || H == 128); }

}  // namespace dsa

using namespace dsa;

#define DSA_SETUP(dev)                                         \
  int dev = 0;                                                 \
  if (!current_device(&dev)) return DSA_ERR_CUDA;              \
  if (!ensure_device(dev)) return DSA_ERR_CUDA;

extern "C" {

dsa_status_t dsa_indexer_scores(const dsa_shape_t* shape, const void* q_idx, const float* q_scale, const void* k_idx,
                                const float* k_scale, const float* w, const int32_t* ctx_len, const int32_t* q_pos0,
                                float* scores, int64_t ld_scores, void* stream) {
  dsa_status_t st = check_shape(shape);
  if (st != DSA_OK) return st;
  st = check_indexer_inputs(shape, q_idx, q_scale, k_idx, k_scale, w, ctx_len, q_pos0);
  if (st != DSA_OK) return st;
  if (!scores || ld_scores < shape->s_max || (ld_scores & 3) != 0 || !aligned16(scores)) return DSA_ERR_INVALID_ARG;
  DSA_SETUP(dev);
  return run_indexer(shape, dev, static_cast<cudaStream_t>(stream), shape->batch, shape->n_q, 0, q_idx, q_scale,
                     k_idx, k_scale, w, ctx_len, q_pos0, scores, ld_scores);
}

dsa_status_t dsa_topk(const dsa_shape_t* shape, const float* scores, int64_t ld_scores, const int32_t* ctx_len,
                      const int32_t* q_pos0, int32_t* idx, void* workspace, size_t workspace_bytes, void* stream) {
  dsa_status_t st = check_shape(shape);
  if (st != DSA_OK) return st;
  if (!scores || !ctx_len || !q_pos0 || !idx) return DSA_ERR_INVALID_ARG;
  if (ld_scores < shape->s_max || (ld_scores & 3) != 0 || !aligned16(scores)) return DSA_ERR_INVALID_ARG;
  const size_t need = topk_workspace_bytes(shape->batch, shape->n_q, shape->s_max, shape->topk);
  if (workspace_bytes < need || (need > 0 && workspace == nullptr)) return DSA_ERR_WORKSPACE;
  DSA_SETUP(dev);
  return run_topk(dev, static_cast<cudaStream_t>(stream), shape->batch, shape->n_q, 0, shape->s_max, shape->topk,
                  scores, ld_scores, ctx_len, q_pos0, idx, workspace, workspace_bytes);
}

dsa_status_t dsa_indexer_proj_q(const dsa_shape_t* shape, int32_t n_tokens, int32_t q_lora_rank,
                                const void* q_latent, const void* wq_b, void* q_idx, void* stream) {
  dsa_status_t st = check_shape(shape);
  if (st != DSA_OK) return st;
  if (n_tokens < 0 || q_lora_rank <= 0) return DSA_ERR_INVALID_ARG;
  if (n_tokens > 0 && (!q_latent || !wq_b || !q_idx)) return DSA_ERR_INVALID_ARG;
  if (!aligned16(q_latent) || !aligned16(wq_b) || !aligned16(q_idx)) return DSA_ERR_INVALID_ARG;
  const int N = shape->idx_heads * shape->idx_dim;
  if (!proj_gemm_supported(N, q_lora_rank, N)) return DSA_ERR_UNSUPPORTED;
  DSA_SETUP(dev);
  GemmArgs a;
  a.device = dev;
  a.stream = static_cast<cudaStream_t>(stream);
  a.M = n_tokens;
  a.N = N;
  a.K = q_lora_rank;
  a.n_split = N;
  a.x = q_latent;
  a.w = wq_b;
  a.out0 = q_idx;
  a.ld0 = N;
  a.out1 = nullptr;
  a.ld1 = 0;
  a.err = g_err_ptr[dev];
  return proj_gemm(a);
}

dsa_status_t dsa_indexer_proj_kw(const dsa_shape_t* shape, int32_t n_tokens, int32_t hidden, const void* x,
                                 const void* w_kw, void* k_new, float* w, void* stream) {
  dsa_status_t st = check_shape(shape);
  if (st != DSA_OK) return st;
  if (n_tokens < 0 || hidden <= 0) return DSA_ERR_INVALID_ARG;
  if (n_tokens > 0 && (!x || !w_kw || !k_new || !w)) return DSA_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(w_kw) || !aligned16(k_new) || !aligned16(w)) return DSA_ERR_INVALID_ARG;
  const int D = shape->idx_dim, HI = shape->idx_heads;
  if ((HI & 3) != 0 || (D & 7) != 0) return DSA_ERR_UNSUPPORTED;
  if (!proj_gemm_supported(D + HI, hidden, D)) return DSA_ERR_UNSUPPORTED;
  DSA_SETUP(dev);
  GemmArgs a;
  a.device = dev;
  a.stream = static_cast<cudaStream_t>(stream);
  a.M = n_tokens;
  a.N = D + HI;
  a.K = hidden;
  a.n_split = D;
  a.x = x;
  a.w = w_kw;
  a.out0 = k_new;
  a.ld0 = D;
  a.out1 = w;
  a.ld1 = HI;
  a.err = g_err_ptr[dev];
  return proj_gemm(a);
}

dsa_status_t dsa_indexer_scores_hist(const dsa_shape_t* shape, const void* q_idx, const float* q_scale,
                                     const void* k_idx, const float* k_scale, const float* w,
                                     const int32_t* ctx_len, const int32_t* q_pos0, float* scores,
                                     int64_t ld_scores, void* hist, size_t hist_bytes, void* stream) {
  dsa_status_t st = check_shape(shape);
  if (st != DSA_OK) return st;
  st = check_indexer_inputs(shape, q_idx, q_scale, k_idx, k_scale, w, ctx_len, q_pos0);
  if (st != DSA_OK) return st;
  if (!scores || ld_scores < shape->s_max || (ld_scores & 3) != 0 || !aligned16(scores)) return DSA_ERR_INVALID_ARG;
  if (hist == nullptr || hist_bytes < kHistPartsBytes || !aligned16(hist)) return DSA_ERR_WORKSPACE;
  DSA_SETUP(dev);
  const HistPlan hp = hist_plan(shape, dev, shape->batch, shape->n_q);
  return run_indexer(shape, dev, static_cast<cudaStream_t>(stream), shape->batch, shape->n_q, 0, q_idx, q_scale,
                     k_idx, k_scale, w, ctx_len, q_pos0, scores, ld_scores,
                     hp.on ? static_cast<uint32_t*>(hist) : nullptr);
}

dsa_status_t dsa_topk_hist(const dsa_shape_t* shape, const float* scores, int64_t ld_scores, const int32_t* ctx_len,
                           const int32_t* q_pos0, const void* hist, size_t hist_bytes, int32_t* idx, void* stream) {
  dsa_status_t st = check_shape(shape);
  if (st != DSA_OK) return st;
  if (!scores || !ctx_len || !q_pos0 || !idx) return DSA_ERR_INVALID_ARG;
  if (ld_scores < shape->s_max || (ld_scores & 3) != 0 || !aligned16(scores)) return DSA_ERR_INVALID_ARG;
  if (hist == nullptr || hist_bytes < kHistPartsBytes) return DSA_ERR_WORKSPACE;
  DSA_SETUP(dev);
  const HistPlan hp = hist_plan(shape, dev, shape->batch, shape->n_q);
  return run_topk(dev, static_cast<cudaStream_t>(stream), shape->batch, shape->n_q, 0, shape->s_max, shape->topk,
                  scores, ld_scores, ctx_len, q_pos0, idx, nullptr, 0, nullptr, 0,
                  hp.on ? static_cast<const uint32_t*>(hist) : nullptr, hp.per_cta, hp.tpr);
}

dsa_status_t dsa_topk_candidates(const dsa_shape_t* shape, const float* cand_scores, const int32_t* cand,
                                 int64_t cand_ld, int32_t n_cand, const int32_t* ctx_len, const int32_t* q_pos0,
                                 int32_t* idx, void* stream) {
  dsa_status_t st = check_shape(shape);
  if (st != DSA_OK) return st;
  if (!cand_scores || !cand || !ctx_len || !q_pos0 || !idx) return DSA_ERR_INVALID_ARG;
  if (n_cand < 0 || cand_ld < n_cand || (cand_ld & 3) != 0 || !aligned16(cand_scores)) return DSA_ERR_INVALID_ARG;
  DSA_SETUP(dev);
  return run_topk(dev, static_cast<cudaStream_t>(stream), shape->batch, shape->n_q, 0, n_cand, shape->topk,
                  cand_scores, cand_ld, ctx_len, q_pos0, idx, nullptr, 0, cand, cand_ld);
}

dsa_status_t dsa_indexer_rescore(const dsa_shape_t* shape, const void* q_idx, const void* k_idx, const float* w,
                                 const int32_t* cand, int64_t cand_ld, int32_t n_cand, const int32_t* ctx_len,
                                 const int32_t* q_pos0, float* scores, int64_t ld_scores, void* stream) {
  dsa_status_t st = check_shape(shape);
  if (st != DSA_OK) return st;
  if (!q_idx || !k_idx || !w || !cand || !ctx_len || !q_pos0 || !scores) return DSA_ERR_INVALID_ARG;
  if (n_cand < 0 || cand_ld < n_cand || ld_scores < n_cand) return DSA_ERR_INVALID_ARG;
  if (!aligned16(q_idx) || !aligned16(k_idx)) return DSA_ERR_INVALID_ARG;
  if (!indexer_rescore_supported(shape->idx_heads, shape->idx_dim)) return DSA_ERR_UNSUPPORTED;
  DSA_SETUP(dev);
  return run_rescore(shape, dev, static_cast<cudaStream_t>(stream), shape->batch, shape->n_q, 0, q_idx, k_idx, w,
                     cand, cand_ld, n_cand, ctx_len, q_pos0, scores, ld_scores);
}

dsa_status_t dsa_sparse_mla_attn(const dsa_shape_t* shape, const void* q, const void* kv, const void* v,
                                 const int32_t* idx, const int32_t* ctx_len, void* out, float* lse, void* workspace,
                                 size_t workspace_bytes, void* stream) {
  dsa_status_t st = check_shape(shape);
  if (st != DSA_OK) return st;
  st = check_attn_inputs(shape, q, kv, v, idx, ctx_len, out);
  if (st != DSA_OK) return st;
  const size_t need = attn_workspace_bytes(shape->batch, shape->n_q, shape->heads, shape->d_qk, shape->d_v,
                                           shape->kv_heads, shape->topk, shape->attn_dtype);
  if (workspace_bytes < need || (need > 0 && workspace == nullptr)) return DSA_ERR_WORKSPACE;
  DSA_SETUP(dev);
  return run_attn(shape, dev, static_cast<cudaStream_t>(stream), shape->batch, shape->n_q, q, kv, v, idx, ctx_len,
                  out, lse, workspace, workspace_bytes);
}

dsa_status_t dsa_cache_append(const dsa_shape_t* shape, int32_t n_new, const void* k_new, const void* kv_new,
                              const void* v_new, const int32_t* pos, void* k_cache, float* k_scale, void* kv_cache,
                              void* v_cache, void* stream) {
  dsa_status_t st = check_shape(shape);
  if (st != DSA_OK) return st;
  if (n_new < 0) return DSA_ERR_INVALID_ARG;
  if (!k_new || !kv_new || !pos || !k_cache || !kv_cache) return DSA_ERR_INVALID_ARG;
  if ((v_new == nullptr) != (v_cache == nullptr)) return DSA_ERR_INVALID_ARG;
  const bool fp8 = shape->idx_dtype == DSA_E4M3;
  if (shape->attn_dtype != DSA_F32 && shape->attn_dtype != DSA_BF16) return DSA_ERR_INVALID_ARG;
  if (fp8 && k_scale == nullptr) return DSA_ERR_INVALID_ARG;
  if (fp8 && shape->idx_dim != 128) return DSA_ERR_UNSUPPORTED;
  const size_t ea = elem_size(shape->attn_dtype);
  AppendArgs a;
  a.k_new = k_new;
  a.kv_new = kv_new;
  a.v_new = v_new;
  a.pos = pos;
  a.k_cache = k_cache;
  a.k_scale = k_scale;
  a.kv_cache = kv_cache;
  a.v_cache = v_cache;
  a.B = shape->batch;
  a.n_new = n_new;
  a.s_max = shape->s_max;
  a.k_row_bytes = fp8 ? 128 : static_cast<int64_t>(shape->idx_dim) * elem_size(shape->idx_dtype);
  a.kv_row_bytes = static_cast<int64_t>(shape->kv_heads) * shape->d_qk * ea;
  a.v_row_bytes = v_new ? static_cast<int64_t>(shape->kv_heads) * shape->d_v * ea : 0;
  // rows are copied in 4-byte words (16-byte chunks when aligned)
  if ((a.k_row_bytes | a.kv_row_bytes | a.v_row_bytes) & 3) return DSA_ERR_UNSUPPORTED;
  const uintptr_t ptrs = reinterpret_cast<uintptr_t>(k_new) | reinterpret_cast<uintptr_t>(kv_new) |
                         reinterpret_cast<uintptr_t>(v_new) | reinterpret_cast<uintptr_t>(k_cache) |
                         reinterpret_cast<uintptr_t>(kv_cache) | reinterpret_cast<uintptr_t>(v_cache) |
                         reinterpret_cast<uintptr_t>(k_scale);
  if (ptrs & 3u) return DSA_ERR_INVALID_ARG;
  DSA_SETUP(dev);
  a.err = g_err_ptr[dev];
  return cache_append(a, fp8, DSA_BF16, static_cast<cudaStream_t>(stream));
}

dsa_status_t dsa_hadamard_quant_fp8(const void* x, int32_t x_dtype, int64_t rows, int32_t dim, uint8_t* x_fp8,
                                    float* scale, void* stream) {
  if (rows < 0 || dim <= 0) return DSA_ERR_INVALID_ARG;
  if (rows > 0 && (!x || !x_fp8 || !scale)) return DSA_ERR_INVALID_ARG;
  if (x_dtype != DSA_BF16 && x_dtype != DSA_F32) return DSA_ERR_INVALID_ARG;
  if (dim != 128) return DSA_ERR_UNSUPPORTED;
  if (((reinterpret_cast<uintptr_t>(x_fp8) & 3u) != 0) || ((reinterpret_cast<uintptr_t>(x) & 7u) != 0))
    return DSA_ERR_INVALID_ARG;
  DSA_SETUP(dev);
  (void)dev;
  return hadamard_quant(x, x_dtype, rows, dim, x_fp8, scale, static_cast<cudaStream_t>(stream));
}

size_t dsa_workspace_bytes(const dsa_shape_t* shape, int32_t which) {
  if (check_shape(shape) != DSA_OK) return 0;
  switch (which) {
    case DSA_WS_TOPK:
      return topk_workspace_bytes(shape->batch, shape->n_q, shape->s_max, shape->topk);
    case DSA_WS_ATTN:
      return attn_workspace_bytes(shape->batch, shape->n_q, shape->heads, shape->d_qk, shape->d_v, shape->kv_heads,
                                  shape->topk, shape->attn_dtype);
    case DSA_WS_FORWARD:
      return forward_layout(shape).total;
    case DSA_WS_FORWARD_HOST:
      return forward_layout(shape).total_host;
    case DSA_WS_HIST:
      return kHistPartsBytes;
    default:
      return 0;
  }
}

// One round of the step over B_ sequences x c queries (pointers already at
// the round's first query; t_off shifts the query positions): indexer
// scores, top-k (the e4m3 indexer with re-scoring: FP8 top-(k + margin)
// candidates, their bf16 scores, then the top-k among them), attention.
struct RoundIn {
  const void* qi;      // indexer queries as the indexer reads them (e4m3 codes or bf16/fp32)
  const float* qsc;    // e4m3 query scales (or null)
  const void* q_ref;   // bf16 queries for re-scoring (or null)
  const void* k_idx;
  const float* k_scale;
  const void* k_ref;   // bf16 key cache for re-scoring (or null)
  const float* w;
  const void* q;
  const void* kv;
  const void* v;
  const int32_t* ctx_len;
  const int32_t* q_pos0;
  void* out;
  float* lse;
  int32_t* idx;
};

static dsa_status_t forward_round(const dsa_shape_t* s, int dev, cudaStream_t st, int B_, int c, int t_off,
                                  const RoundIn& in, uint8_t* ws, const FwdLayout& L, cudaEvent_t q_ready,
                                  cudaEvent_t out_free) {
  float* scores = reinterpret_cast<float*>(ws + L.off_scores);
  // decode: the indexer's epilogue also counts the first radix digit of each
  // score row, so the top-k starts from the threshold bin
  const HistPlan hp = (L.chunk == 1) ? hist_plan(s, dev, B_, c) : HistPlan{};
  uint32_t* hist = hp.on ? reinterpret_cast<uint32_t*>(ws + L.off_hist) : nullptr;
  dsa_status_t rc = run_indexer(s, dev, st, B_, c, t_off, in.qi, in.qsc, in.k_idx, in.k_scale, in.w, in.ctx_len,
                                in.q_pos0, scores, L.ld, hist);
  if (rc != DSA_OK) return rc;
  if (L.kc > 0) {
    int32_t* cand = reinterpret_cast<int32_t*>(ws + L.off_cand);
    float* rs = reinterpret_cast<float*>(ws + L.off_rs);
    rc = run_topk(dev, st, B_, c, t_off, s->s_max, L.kc, scores, L.ld, in.ctx_len, in.q_pos0, cand,
                  ws + L.off_topk, L.topk_bytes, nullptr, 0, hist, hp.per_cta, hp.tpr);
    if (rc != DSA_OK) return rc;
    rc = run_rescore(s, dev, st, B_, c, t_off, in.q_ref, in.k_ref, in.w, cand, L.kc, L.kc, in.ctx_len, in.q_pos0,
                     rs, L.kc);
    if (rc != DSA_OK) return rc;
    rc = run_topk(dev, st, B_, c, t_off, L.kc, s->topk, rs, L.kc, in.ctx_len, in.q_pos0, in.idx, ws + L.off_topk,
                  L.topk_bytes, cand, L.kc);
  } else {
    rc = run_topk(dev, st, B_, c, t_off, s->s_max, s->topk, scores, L.ld, in.ctx_len, in.q_pos0, in.idx,
                  ws + L.off_topk, L.topk_bytes, nullptr, 0, hist, hp.per_cta, hp.tpr);
  }
  if (rc != DSA_OK) return rc;
  if (q_ready != nullptr && cudaStreamWaitEvent(st, q_ready, 0) != cudaSuccess) return DSA_ERR_CUDA;
  if (out_free != nullptr && cudaStreamWaitEvent(st, out_free, 0) != cudaSuccess) return DSA_ERR_CUDA;
  return run_attn(s, dev, st, B_, c, in.q, in.kv, in.v, in.idx, in.ctx_len, in.out, in.lse, ws + L.off_attn,
                  L.attn_bytes);
}

static dsa_status_t forward_impl(const dsa_shape_t* s, int dev, cudaStream_t st, const void* q_idx,
                                 const float* q_scale, const void* k_idx, const float* k_scale, const void* k_ref,
                                 const float* w, const void* q, const void* kv, const void* v,
                                 const int32_t* ctx_len, const int32_t* q_pos0, void* out, float* lse,
                                 int32_t* idx_out, uint8_t* ws, const FwdLayout& L, cudaEvent_t q_ready = nullptr,
                                 cudaEvent_t out_free = nullptr) {
  const int B = s->batch, n_q = s->n_q;
  if (B == 0 || n_q == 0) return DSA_OK;
  dsa_status_t rc;
  // FP8 indexer: rotate + quantise this step's queries
  const void* qi = q_idx;
  const float* qsc = q_scale;
  if (s->idx_dtype == DSA_E4M3) {
    rc = hadamard_quant(q_idx, DSA_BF16, static_cast<int64_t>(B) * n_q * s->idx_heads, s->idx_dim, ws + L.off_q8,
                        reinterpret_cast<float*>(ws + L.off_qs), st);
    if (rc != DSA_OK) return rc;
    qi = ws + L.off_q8;
    qsc = reinterpret_cast<float*>(ws + L.off_qs);
  }
  const size_t ei = elem_size(s->idx_dtype);
  const size_t ea = elem_size(s->attn_dtype);
  RoundIn in;
  if (L.chunk == n_q) {
    in = {qi, qsc, q_idx, k_idx, k_scale, k_ref, w, q, kv, v, ctx_len, q_pos0, out, lse,
          idx_out ? idx_out : reinterpret_cast<int32_t*>(ws + L.off_idx)};
    return forward_round(s, dev, st, B, n_q, 0, in, ws, L, q_ready, out_free);
  }
  // Rounds of `chunk` queries, one sequence at a time (positions shift by t0).
  const int64_t qrow = static_cast<int64_t>(s->idx_heads) * s->idx_dim;
  for (int b = 0; b < B; ++b) {
    for (int t0 = 0; t0 < n_q; t0 += L.chunk) {
      const int c = std::min(L.chunk, n_q - t0);
      const int64_t row0 = static_cast<int64_t>(b) * n_q + t0;
      in.qi = static_cast<const uint8_t*>(qi) + row0 * qrow * ei;
      in.qsc = qsc ? qsc + row0 * s->idx_heads : nullptr;
      in.q_ref = static_cast<const uint8_t*>(q_idx) + row0 * qrow * 2;
      in.k_idx = static_cast<const uint8_t*>(k_idx) + static_cast<int64_t>(b) * s->s_max * s->idx_dim * ei;
      in.k_scale = k_scale ? k_scale + static_cast<int64_t>(b) * s->s_max : nullptr;
      in.k_ref = k_ref ? static_cast<const uint8_t*>(k_ref) + static_cast<int64_t>(b) * s->s_max * s->idx_dim * 2
                       : nullptr;
      in.w = w + row0 * s->idx_heads;
      in.q = static_cast<const uint8_t*>(q) + row0 * s->heads * s->d_qk * ea;
      in.kv = static_cast<const uint8_t*>(kv) + static_cast<int64_t>(b) * s->s_max * s->kv_heads * s->d_qk * ea;
      in.v = v ? static_cast<const uint8_t*>(v) + static_cast<int64_t>(b) * s->s_max * s->kv_heads * s->d_v * ea
               : nullptr;
      in.ctx_len = ctx_len + b;
      in.q_pos0 = q_pos0 + b;
      in.out = static_cast<uint8_t*>(out) + row0 * s->heads * s->d_v * ea;
      in.lse = lse ? lse + row0 * s->heads : nullptr;
      in.idx = idx_out ? idx_out + row0 * s->topk : reinterpret_cast<int32_t*>(ws + L.off_idx);
      const bool first = (b == 0 && t0 == 0);
      rc = forward_round(s, dev, st, 1, c, t0, in, ws, L, first ? q_ready : nullptr, first ? out_free : nullptr);
      if (rc != DSA_OK) return rc;
    }
  }
  return DSA_OK;
}

static dsa_status_t check_forward(const dsa_shape_t* shape, const void* q_idx, const float* q_scale,
                                  const void* k_idx, const float* k_scale, const void* k_ref, const float* w,
                                  const void* q, const void* kv, const void* v, const int32_t* ctx_len,
                                  const int32_t* q_pos0, const void* out, bool on_host) {
  dsa_status_t st = check_shape(shape);
  if (st != DSA_OK) return st;
  if (shape->idx_dtype == DSA_E4M3) {
    if (q_scale != nullptr || !k_scale || !q_idx || !k_idx || !w || !ctx_len || !q_pos0) return DSA_ERR_INVALID_ARG;
    if (!aligned16(k_idx) || (!on_host && !aligned16(q_idx))) return DSA_ERR_INVALID_ARG;
    if (!indexer_tc_supported(shape->idx_heads, shape->idx_dim)) return DSA_ERR_UNSUPPORTED;
    if (shape->idx_rescore > 0) {
      if (!k_ref || !aligned16(k_ref)) return DSA_ERR_INVALID_ARG;
      if (!indexer_rescore_supported(shape->idx_heads, shape->idx_dim)) return DSA_ERR_UNSUPPORTED;
    } else if (k_ref != nullptr) {
      return DSA_ERR_INVALID_ARG;
    }
  } else {
    if (k_ref != nullptr) return DSA_ERR_INVALID_ARG;
    if (!on_host) {
      st = check_indexer_inputs(shape, q_idx, q_scale, k_idx, k_scale, w, ctx_len, q_pos0);
      if (st != DSA_OK) return st;
    } else if (!q_idx || !k_idx || !w || !ctx_len || !q_pos0) {
      return DSA_ERR_INVALID_ARG;
    }
  }
  if (!q || !kv || !out) return DSA_ERR_INVALID_ARG;
  if (!on_host) {
    st = check_attn_inputs(shape, q, kv, v, /*idx*/ q, ctx_len, out);
    if (st != DSA_OK) return st;
  }
  return DSA_OK;
}

dsa_status_t dsa_forward(const dsa_shape_t* shape, const void* q_idx, const float* q_scale, const void* k_idx,
                         const float* k_scale, const void* k_rescore, const float* w, const void* q, const void* kv,
                         const void* v, const int32_t* ctx_len, const int32_t* q_pos0, void* out, float* lse,
                         int32_t* idx_out, void* workspace, size_t workspace_bytes, void* stream) {
  dsa_status_t st = check_forward(shape, q_idx, q_scale, k_idx, k_scale, k_rescore, w, q, kv, v, ctx_len, q_pos0,
                                  out, false);
  if (st != DSA_OK) return st;
  const FwdLayout L = forward_layout(shape);
  if (workspace == nullptr || workspace_bytes < L.total || !aligned16(workspace)) return DSA_ERR_WORKSPACE;
  DSA_SETUP(dev);
  return forward_impl(shape, dev, static_cast<cudaStream_t>(stream), q_idx, q_scale, k_idx, k_scale, k_rescore, w, q,
                      kv, v, ctx_len, q_pos0, out, lse, idx_out, static_cast<uint8_t*>(workspace), L);
}

// The step with host-memory inputs and outputs.  Synchronous: the output is
// copied back on the compute stream and the call returns after it.
// Asynchronous: the output is copied back on the library's output stream
// after the attention, `done` (if given) is recorded after that copy, and the
// call returns once everything is enqueued; the next call's attention waits
// for the copy before it rewrites the device output.
static dsa_status_t forward_host_impl(const dsa_shape_t* shape, const void* h_q_idx, const float* h_w,
                                      const void* h_q, const int32_t* h_ctx_len, const int32_t* h_q_pos0,
                                      const void* k_idx, const float* k_scale, const void* k_rescore,
                                      const void* kv, const void* v,
                                      void* h_out, float* h_lse, void* workspace, size_t workspace_bytes,
                                      void* stream, bool async, cudaEvent_t done) {
  dsa_status_t st = check_forward(shape, h_q_idx, nullptr, k_idx, k_scale, k_rescore, h_w, h_q, kv, v, h_ctx_len,
                                  h_q_pos0, h_out, true);
  if (st != DSA_OK) return st;
  const FwdLayout L = forward_layout(shape);
  if (workspace == nullptr || workspace_bytes < L.total_host || !aligned16(workspace)) return DSA_ERR_WORKSPACE;
  DSA_SETUP(dev);
  const cudaStream_t cs = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const int B = shape->batch, n_q = shape->n_q;
  const size_t ai = elem_size(shape->idx_dtype == DSA_E4M3 ? DSA_BF16 : shape->idx_dtype);
  const size_t aa = elem_size(shape->attn_dtype);
  const size_t n_qidx = static_cast<size_t>(B) * n_q * shape->idx_heads * shape->idx_dim * ai;
  const size_t n_w = static_cast<size_t>(B) * n_q * shape->idx_heads * 4;
  const size_t n_q_b = static_cast<size_t>(B) * n_q * shape->heads * shape->d_qk * aa;
  const size_t n_out = static_cast<size_t>(B) * n_q * shape->heads * shape->d_v * aa;
  const size_t n_lse = static_cast<size_t>(B) * n_q * shape->heads * 4;
  // inputs travel on the copy stream into this call's slot, once the last
  // call that used the slot has finished its attention: the indexer inputs
  // first (the compute stream waits for them), then the attention queries
  // (the bulk of the input: waited for just before attention, so that they
  // land under the indexer and top-k)
  if (!ensure_copy_stream(dev)) return DSA_ERR_CUDA;
  std::lock_guard<std::mutex> host_lock(g_host_mutex[dev]);
  const cudaStream_t xs = g_copy_stream[dev];
  const int slot = g_slot[dev];
  g_slot[dev] ^= 1;
  uint8_t* in = ws + L.off_h_in[slot];
  if (g_last_ws[dev] != workspace) {
    if (cudaEventRecord(g_ev_join[dev], cs) != cudaSuccess || cudaStreamWaitEvent(xs, g_ev_join[dev], 0) != cudaSuccess)
      return DSA_ERR_CUDA;
    g_last_ws[dev] = workspace;
  }
  if (cudaStreamWaitEvent(xs, g_ev_free[dev][slot], 0) != cudaSuccess ||
      cudaMemcpyAsync(in + L.off_h_qidx, h_q_idx, n_qidx, cudaMemcpyHostToDevice, xs) != cudaSuccess ||
      cudaMemcpyAsync(in + L.off_h_w, h_w, n_w, cudaMemcpyHostToDevice, xs) != cudaSuccess ||
      cudaMemcpyAsync(in + L.off_h_ctx, h_ctx_len, static_cast<size_t>(B) * 4, cudaMemcpyHostToDevice, xs) !=
          cudaSuccess ||
      cudaMemcpyAsync(in + L.off_h_pos, h_q_pos0, static_cast<size_t>(B) * 4, cudaMemcpyHostToDevice, xs) !=
          cudaSuccess ||
      cudaEventRecord(g_ev_in[dev], xs) != cudaSuccess ||
      cudaMemcpyAsync(in + L.off_h_q, h_q, n_q_b, cudaMemcpyHostToDevice, xs) != cudaSuccess ||
      cudaEventRecord(g_ev_q[dev], xs) != cudaSuccess || cudaStreamWaitEvent(cs, g_ev_in[dev], 0) != cudaSuccess)
    return DSA_ERR_CUDA;
  dsa_shape_t s2 = *shape;
  st = forward_impl(&s2, dev, cs, in + L.off_h_qidx, nullptr, k_idx, k_scale, k_rescore,
                    reinterpret_cast<float*>(in + L.off_h_w),
                    in + L.off_h_q, kv, v, reinterpret_cast<int32_t*>(in + L.off_h_ctx),
                    reinterpret_cast<int32_t*>(in + L.off_h_pos), ws + L.off_h_out,
                    h_lse ? reinterpret_cast<float*>(ws + L.off_h_lse) : nullptr, nullptr, ws, L, g_ev_q[dev],
                    g_ev_out[dev]);
  // (already waited before attention; again here so that no copy into the
  // workspace is left in flight on any path)
  if (cudaStreamWaitEvent(cs, g_ev_q[dev], 0) != cudaSuccess && st == DSA_OK) st = DSA_ERR_CUDA;
  if (cudaStreamWaitEvent(cs, g_ev_out[dev], 0) != cudaSuccess && st == DSA_OK) st = DSA_ERR_CUDA;
  // the slot is free once everything enqueued so far has run, on the error
  // paths too (kernels enqueued before a failure may still read it)
  if (cudaEventRecord(g_ev_free[dev][slot], cs) != cudaSuccess && st == DSA_OK) st = DSA_ERR_CUDA;
  if (st != DSA_OK) return st;
  const cudaStream_t os = async ? g_out_stream[dev] : cs;
  if (async && (cudaEventRecord(g_ev_attn[dev], cs) != cudaSuccess ||
                cudaStreamWaitEvent(os, g_ev_attn[dev], 0) != cudaSuccess))
    return DSA_ERR_CUDA;
  if (cudaMemcpyAsync(h_out, ws + L.off_h_out, n_out, cudaMemcpyDeviceToHost, os) != cudaSuccess) return DSA_ERR_CUDA;
  if (h_lse && cudaMemcpyAsync(h_lse, ws + L.off_h_lse, n_lse, cudaMemcpyDeviceToHost, os) != cudaSuccess)
    return DSA_ERR_CUDA;
  if (!async) return cudaStreamSynchronize(cs) == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
  if (cudaEventRecord(g_ev_out[dev], os) != cudaSuccess) return DSA_ERR_CUDA;
  if (done != nullptr && cudaEventRecord(done, os) != cudaSuccess) return DSA_ERR_CUDA;
  return DSA_OK;
}

dsa_status_t dsa_forward_host(const dsa_shape_t* shape, const void* h_q_idx, const float* h_w, const void* h_q,
                              const int32_t* h_ctx_len, const int32_t* h_q_pos0, const void* k_idx,
                              const float* k_scale, const void* k_rescore, const void* kv, const void* v,
                              void* h_out, float* h_lse, void* workspace, size_t workspace_bytes, void* stream) {
  return forward_host_impl(shape, h_q_idx, h_w, h_q, h_ctx_len, h_q_pos0, k_idx, k_scale, k_rescore, kv, v, h_out,
                           h_lse,
                           workspace, workspace_bytes, stream, false, nullptr);
}

dsa_status_t dsa_forward_host_async(const dsa_shape_t* shape, const void* h_q_idx, const float* h_w,
                                    const void* h_q, const int32_t* h_ctx_len, const int32_t* h_q_pos0,
                                    const void* k_idx, const float* k_scale, const void* k_rescore, const void* kv,
                                    const void* v, void* h_out, float* h_lse, void* workspace,
                                    size_t workspace_bytes, void* done_event, void* stream) {
  return forward_host_impl(shape, h_q_idx, h_w, h_q, h_ctx_len, h_q_pos0, k_idx, k_scale, k_rescore, kv, v, h_out,
                           h_lse,
                           workspace, workspace_bytes, stream, true, static_cast<cudaEvent_t>(done_event));
}

dsa_status_t dsa_get_error(int32_t clear, uint32_t* detail) {
  DSA_SETUP(dev);
  uint32_t word[4] = {0, 0, 0, 0};
  if (cudaDeviceSynchronize() != cudaSuccess) return DSA_ERR_CUDA;
  if (cudaMemcpy(word, g_err_ptr[dev], sizeof(word), cudaMemcpyDeviceToHost) != cudaSuccess) return DSA_ERR_CUDA;
  if (clear) {
    const uint32_t zero[4] = {0, 0, 0, 0};
    if (cudaMemcpy(g_err_ptr[dev], zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess) return DSA_ERR_CUDA;
  }
  if (detail) *detail = word[0];
  if (word[0] & kErrTimeout) return DSA_ERR_TIMEOUT;
  if (word[0] & kErrBadIndex) return DSA_ERR_BAD_INDEX;
  if (word[0] & kErrHistMismatch) return DSA_ERR_HIST_MISMATCH;
  return DSA_OK;
}

const char* dsa_status_string(dsa_status_t status) {
  switch (status) {
    case DSA_OK: return "ok";
    case DSA_ERR_INVALID_ARG: return "invalid argument";
    case DSA_ERR_UNSUPPORTED: return "unsupported shape or dtype";
    case DSA_ERR_WORKSPACE: return "workspace missing or too small";
    case DSA_ERR_CUDA: return "CUDA error";
    case DSA_ERR_TIMEOUT: return "a bounded wait inside a kernel expired";
    case DSA_ERR_BAD_INDEX: return "attention index out of range (skipped)";
    case DSA_ERR_HIST_MISMATCH: return "handed-over histograms do not match the scores";
  }
  return "unknown status";
}

int32_t dsa_version(void) { return 100; }

dsa_status_t dsa_selftest_wait_timeout(void* stream) {
  DSA_SETUP(dev);
  return selftest_wait_timeout(g_err_ptr[dev], static_cast<cudaStream_t>(stream));
}

}  // extern "C"

// ------------------------------------------------ allocation-free attention --
// dsa_sparse_mla_attn_static: the same attention, with the scratch memory of
// the split-K combine taken from a fixed array inside this library instead
// of a caller-provided workspace.  For callers that cannot hand the library
// device memory on their decode path: a serving loop whose device memory is
// planned once up front and may not grow, or a host program with no device
// allocator of its own -- for both, cudaMalloc is also a poor fit because it
// can synchronise the whole device.
namespace dsa {
namespace {

// Capacity of the scratch array.  A 148-SM B200 needs at most about 20 MB
// (decode with 37 queries per call); larger needs are rejected.
constexpr size_t kStaticAttnScratchBytes = size_t(32) << 20;

// File-scope device array: every GPU that loads this library holds it until
// the process exits.  Host code must not pass `g_attn_scratch` itself to a
// kernel -- in host code the name is a stand-in, not a device address -- but
// the address obtained with cudaGetSymbolAddress below.
__device__ __align__(256) unsigned char g_attn_scratch[kStaticAttnScratchBytes];

std::mutex g_static_mutex;
void* g_static_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on `dev` (the current device), looked
// up once per device.
void* static_attn_scratch(int dev) {
  std::lock_guard<std::mutex> lock(g_static_mutex);
  if (g_static_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_attn_scratch) != cudaSuccess) {
      (void)cudaGetLastError();  // consumed here, so it is not reported against a later call
      return nullptr;
    }
    g_static_scratch_ptr[dev] = p;
  }
  return g_static_scratch_ptr[dev];
}

}  // namespace
}  // namespace dsa

extern "C" dsa_status_t dsa_sparse_mla_attn_static(const dsa_shape_t* shape, const void* q, const void* kv,
                                                   const void* v, const int32_t* idx, const int32_t* ctx_len,
                                                   void* out, float* lse, void* stream) {
  dsa_status_t st = check_shape(shape);
  if (st != DSA_OK) return st;
  st = check_attn_inputs(shape, q, kv, v, idx, ctx_len, out);
  if (st != DSA_OK) return st;
  DSA_SETUP(dev);
  size_t need = 0;
  if (shape->attn_dtype == DSA_BF16 && attn_tc_supported(shape->heads, shape->d_qk, shape->d_v, shape->kv_heads))
    need = attn_scratch_bytes(shape->batch, shape->n_q, shape->topk, device_sm_count(dev));
  if (need > kStaticAttnScratchBytes) return DSA_ERR_WORKSPACE;  // beyond the fixed capacity
  void* scratch = static_attn_scratch(dev);
  if (scratch == nullptr) return DSA_ERR_CUDA;
  return run_attn(shape, dev, static_cast<cudaStream_t>(stream), shape->batch, shape->n_q, q, kv, v, idx, ctx_len,
                  out, lse, scratch, kStaticAttnScratchBytes);
}
