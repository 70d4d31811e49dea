"""Python binding of libdsa.so -- the DeepSeek Sparse Attention (DSA) layer
step on one B200: Lightning-indexer scores, causal top-k selection, and MLA
attention over the selected latent rows (DeepSeek-V3.2 model doc,
Transformers, section "DeepSeek Sparse Attention (DSA)").

This module only marshals arguments: torch tensors supply device memory and
the current CUDA stream; every step runs in the library's CUDA kernels.  If
the library is missing, importing the functions raises -- there is no CPU
path.  Names and argument order follow ``include/dsa.h``.
"""
import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libdsa.so")

DSA_F32, DSA_BF16, DSA_E4M3 = 0, 1, 2
WS_TOPK, WS_ATTN, WS_FORWARD, WS_FORWARD_HOST, WS_HIST = 0, 1, 2, 3, 4

STATUS = {
    0: "DSA_OK", 1: "DSA_ERR_INVALID_ARG", 2: "DSA_ERR_UNSUPPORTED", 3: "DSA_ERR_WORKSPACE",
    4: "DSA_ERR_CUDA", 5: "DSA_ERR_TIMEOUT", 6: "DSA_ERR_BAD_INDEX", 7: "DSA_ERR_HIST_MISMATCH",
}

EXPORTS = (
    "dsa_indexer_scores", "dsa_topk", "dsa_sparse_mla_attn", "dsa_hadamard_quant_fp8", "dsa_cache_append",
    "dsa_forward",
    "dsa_forward_host", "dsa_forward_host_async", "dsa_workspace_bytes", "dsa_get_error", "dsa_status_string", "dsa_version",
    "dsa_sparse_mla_attn_static", "dsa_selftest_wait_timeout", "dsa_indexer_rescore", "dsa_topk_candidates",
    "dsa_indexer_scores_hist", "dsa_topk_hist", "dsa_indexer_proj_q", "dsa_indexer_proj_kw",
)


class DsaError(RuntimeError):
    def __init__(self, status, where):
        self.status = status
        super().__init__(f"{where}: {STATUS.get(status, status)}")


class Shape(ctypes.Structure):
    """Mirror of ``dsa_shape_t``."""
    _fields_ = [
        ("batch", ctypes.c_int32), ("n_q", ctypes.c_int32), ("s_max", ctypes.c_int32),
        ("idx_heads", ctypes.c_int32), ("idx_dim", ctypes.c_int32), ("topk", ctypes.c_int32),
        ("heads", ctypes.c_int32), ("d_qk", ctypes.c_int32), ("d_v", ctypes.c_int32),
        ("kv_heads", ctypes.c_int32), ("idx_dtype", ctypes.c_int32), ("attn_dtype", ctypes.c_int32),
        ("idx_scale", ctypes.c_float), ("sm_scale", ctypes.c_float), ("q_chunk", ctypes.c_int32),
        ("idx_rescore", ctypes.c_int32),
    ]

    def replace(self, **kw):
        s = Shape()
        ctypes.pointer(s)[0] = self
        for k, v in kw.items():
            setattr(s, k, v)
        return s


_lib = None


def lib():
    """Load libdsa.so (built in-tree by ``build.py``); raises if it is absent."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"libdsa.so not built ({LIB_PATH}); run python -m long_context_indexing_lightning_b200.build")
        L = ctypes.CDLL(LIB_PATH)
        P, S = ctypes.c_void_p, ctypes.POINTER(Shape)
        i32, i64, sz = ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
        L.dsa_indexer_scores.argtypes = [S, P, P, P, P, P, P, P, P, i64, P]
        L.dsa_topk.argtypes = [S, P, i64, P, P, P, P, sz, P]
        L.dsa_sparse_mla_attn.argtypes = [S, P, P, P, P, P, P, P, P, sz, P]
        L.dsa_hadamard_quant_fp8.argtypes = [P, i32, i64, i32, P, P, P]
        L.dsa_cache_append.argtypes = [S, i32, P, P, P, P, P, P, P, P, P]
        L.dsa_sparse_mla_attn_static.argtypes = [S, P, P, P, P, P, P, P, P]
        L.dsa_selftest_wait_timeout.argtypes = [P]
        L.dsa_forward.argtypes = [S, P, P, P, P, P, P, P, P, P, P, P, P, P, P, P, sz, P]
        L.dsa_forward_host.argtypes = [S, P, P, P, P, P, P, P, P, P, P, P, P, P, sz, P]
        L.dsa_forward_host_async.argtypes = [S, P, P, P, P, P, P, P, P, P, P, P, P, P, sz, P, P]
        L.dsa_indexer_rescore.argtypes = [S, P, P, P, P, i64, i32, P, P, P, i64, P]
        L.dsa_topk_candidates.argtypes = [S, P, P, i64, i32, P, P, P, P]
        L.dsa_indexer_scores_hist.argtypes = [S, P, P, P, P, P, P, P, P, i64, P, sz, P]
        L.dsa_topk_hist.argtypes = [S, P, i64, P, P, P, sz, P, P]
        L.dsa_indexer_proj_q.argtypes = [S, i32, i32, P, P, P, P]
        L.dsa_indexer_proj_kw.argtypes = [S, i32, i32, P, P, P, P, P]
        L.dsa_workspace_bytes.argtypes = [S, i32]
        L.dsa_workspace_bytes.restype = sz
        L.dsa_get_error.argtypes = [i32, ctypes.POINTER(ctypes.c_uint32)]
        L.dsa_status_string.argtypes = [i32]
        L.dsa_status_string.restype = ctypes.c_char_p
        L.dsa_version.restype = i32
        for name in EXPORTS:
            if name not in ("dsa_workspace_bytes", "dsa_status_string", "dsa_version"):
                getattr(L, name).restype = i32
        _lib = L
    return _lib


def _p(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _check(rc, where):
    if rc != 0:
        raise DsaError(rc, where)


def _dtype_code(t: torch.dtype) -> int:
    return {torch.float32: DSA_F32, torch.bfloat16: DSA_BF16, torch.uint8: DSA_E4M3}[t]


def make_shape(batch, n_q, s_max, idx_heads=64, idx_dim=128, topk=2048, heads=128, d_qk=576, d_v=512,
               kv_heads=1, idx_dtype=DSA_BF16, attn_dtype=DSA_BF16, idx_scale=1.0, sm_scale=None,
               q_chunk=0, idx_rescore=0) -> Shape:
    if sm_scale is None:
        sm_scale = (192 ** -0.5) if kv_heads == 1 else d_qk ** -0.5
    return Shape(batch, n_q, s_max, idx_heads, idx_dim, topk, heads, d_qk, d_v, kv_heads, idx_dtype,
                 attn_dtype, float(idx_scale), float(sm_scale), q_chunk, idx_rescore)


def shape_from_workload(wl, q_chunk=0) -> Shape:
    """Shape for a ``workloads.Workload`` (duck-typed: reads its fields)."""
    dt = DSA_BF16 if wl.dtype == "bf16" else DSA_F32
    return make_shape(wl.batch, wl.n_q, wl.s_max, wl.idx_heads, wl.idx_dim, wl.topk, wl.heads, wl.d_qk, wl.d_v,
                      wl.kv_heads, DSA_E4M3 if wl.idx_fp8 else dt, dt, wl.idx_scale, wl.sm_scale, q_chunk,
                      wl.idx_rescore if wl.idx_fp8 else 0)


def workspace_bytes(shape: Shape, which: int) -> int:
    return int(lib().dsa_workspace_bytes(ctypes.byref(shape), which))


def _workspace(shape, which, ws, device):
    n = workspace_bytes(shape, which)
    if ws is None and n > 0:
        ws = torch.empty(n, dtype=torch.uint8, device=device)
    return ws, (ws.numel() if ws is not None else 0)


def indexer_scores(shape, q_idx, k_idx, w, ctx_len, q_pos0, scores=None, q_scale=None, k_scale=None, ld=None,
                   stream=None):
    """Scores [B, n_q, ld] fp32 (see dsa_indexer_scores)."""
    if scores is None:
        ld = ld or ((shape.s_max + 3) // 4 * 4)
        scores = torch.empty(shape.batch, shape.n_q, ld, dtype=torch.float32, device=k_idx.device)
    ld = scores.stride(1) if scores.dim() == 3 else scores.stride(0)
    _check(lib().dsa_indexer_scores(ctypes.byref(shape), _p(q_idx), _p(q_scale), _p(k_idx), _p(k_scale), _p(w),
                                    _p(ctx_len), _p(q_pos0), _p(scores), ld, _stream(stream)),
           "dsa_indexer_scores")
    return scores


def topk(shape, scores, ctx_len, q_pos0, idx=None, workspace=None, stream=None):
    """Indices [B, n_q, topk] int32, ascending then -1 (see dsa_topk)."""
    if idx is None:
        idx = torch.empty(shape.batch, shape.n_q, shape.topk, dtype=torch.int32, device=scores.device)
    ws, n = _workspace(shape, WS_TOPK, workspace, scores.device)
    ld = scores.stride(1) if scores.dim() == 3 else scores.stride(0)
    _check(lib().dsa_topk(ctypes.byref(shape), _p(scores), ld, _p(ctx_len), _p(q_pos0), _p(idx), _p(ws), n,
                          _stream(stream)), "dsa_topk")
    return idx


def indexer_proj_q(shape, q_latent, wq_b, q_idx=None, stream=None):
    """Index queries [T, H_I, D_I] bf16 from the query latent [T, q_lora_rank] (see dsa_indexer_proj_q)."""
    T, r = q_latent.shape[0], q_latent.shape[-1]
    if q_idx is None:
        q_idx = torch.empty(T, shape.idx_heads, shape.idx_dim, dtype=torch.bfloat16, device=q_latent.device)
    _check(lib().dsa_indexer_proj_q(ctypes.byref(shape), T, r, _p(q_latent), _p(wq_b), _p(q_idx),
                                    _stream(stream)), "dsa_indexer_proj_q")
    return q_idx


def indexer_proj_kw(shape, x, w_kw, k_new=None, w=None, stream=None):
    """Index keys [T, D_I] bf16 and head weights [T, H_I] fp32 from the hidden state (see dsa_indexer_proj_kw)."""
    T, hidden = x.shape[0], x.shape[-1]
    if k_new is None:
        k_new = torch.empty(T, shape.idx_dim, dtype=torch.bfloat16, device=x.device)
    if w is None:
        w = torch.empty(T, shape.idx_heads, dtype=torch.float32, device=x.device)
    _check(lib().dsa_indexer_proj_kw(ctypes.byref(shape), T, hidden, _p(x), _p(w_kw), _p(k_new), _p(w),
                                     _stream(stream)), "dsa_indexer_proj_kw")
    return k_new, w


def indexer_scores_hist(shape, q_idx, k_idx, w, ctx_len, q_pos0, hist, scores=None, q_scale=None, k_scale=None,
                        stream=None):
    """Scores as indexer_scores, also filling the top-k handoff `hist` (see dsa_indexer_scores_hist)."""
    if scores is None:
        ld = (shape.s_max + 3) // 4 * 4
        scores = torch.empty(shape.batch, shape.n_q, ld, dtype=torch.float32, device=k_idx.device)
    ld = scores.stride(1) if scores.dim() == 3 else scores.stride(0)
    _check(lib().dsa_indexer_scores_hist(ctypes.byref(shape), _p(q_idx), _p(q_scale), _p(k_idx), _p(k_scale),
                                         _p(w), _p(ctx_len), _p(q_pos0), _p(scores), ld, _p(hist),
                                         hist.numel() * hist.element_size(), _stream(stream)),
           "dsa_indexer_scores_hist")
    return scores


def topk_hist(shape, scores, ctx_len, q_pos0, hist, idx=None, stream=None):
    """Top-k as topk, starting from the indexer's handoff `hist` (see dsa_topk_hist)."""
    if idx is None:
        idx = torch.empty(shape.batch, shape.n_q, shape.topk, dtype=torch.int32, device=scores.device)
    ld = scores.stride(1) if scores.dim() == 3 else scores.stride(0)
    _check(lib().dsa_topk_hist(ctypes.byref(shape), _p(scores), ld, _p(ctx_len), _p(q_pos0), _p(hist),
                               hist.numel() * hist.element_size(), _p(idx), _stream(stream)), "dsa_topk_hist")
    return idx


def topk_candidates(shape, cand_scores, cand, n_cand, ctx_len, q_pos0, idx=None, stream=None):
    """Top-k among listed candidates [B, n_q, cand_ld] (see dsa_topk_candidates)."""
    if idx is None:
        idx = torch.empty(shape.batch, shape.n_q, shape.topk, dtype=torch.int32, device=cand.device)
    ld = cand.stride(1) if cand.dim() == 3 else cand.stride(0)
    if cand_scores.stride(1 if cand_scores.dim() == 3 else 0) != ld:
        raise ValueError("cand_scores and cand must share their row stride")
    _check(lib().dsa_topk_candidates(ctypes.byref(shape), _p(cand_scores), _p(cand), ld, int(n_cand), _p(ctx_len),
                                     _p(q_pos0), _p(idx), _stream(stream)), "dsa_topk_candidates")
    return idx


def indexer_rescore(shape, q_idx, k_idx, w, cand, n_cand, ctx_len, q_pos0, scores=None, stream=None):
    """BF16 index scores of listed keys [B, n_q, >= n_cand] fp32 (see dsa_indexer_rescore)."""
    cand_ld = cand.stride(1) if cand.dim() == 3 else cand.stride(0)
    if scores is None:
        scores = torch.empty(shape.batch, shape.n_q, max(1, int(n_cand)), dtype=torch.float32, device=k_idx.device)
    ld = scores.stride(1) if scores.dim() == 3 else scores.stride(0)
    _check(lib().dsa_indexer_rescore(ctypes.byref(shape), _p(q_idx), _p(k_idx), _p(w), _p(cand), cand_ld,
                                     int(n_cand), _p(ctx_len), _p(q_pos0), _p(scores), ld, _stream(stream)),
           "dsa_indexer_rescore")
    return scores


def sparse_mla_attn(shape, q, kv, idx, ctx_len, out=None, v=None, lse=None, workspace=None, stream=None):
    """Attention output [B, n_q, H, d_v] (see dsa_sparse_mla_attn)."""
    if out is None:
        out = torch.empty(shape.batch, shape.n_q, shape.heads, shape.d_v, dtype=q.dtype, device=q.device)
    ws, n = _workspace(shape, WS_ATTN, workspace, q.device)
    _check(lib().dsa_sparse_mla_attn(ctypes.byref(shape), _p(q), _p(kv), _p(v), _p(idx), _p(ctx_len), _p(out),
                                     _p(lse), _p(ws), n, _stream(stream)), "dsa_sparse_mla_attn")
    return out


def sparse_mla_attn_static(shape, q, kv, idx, ctx_len, out=None, v=None, lse=None, stream=None):
    """As sparse_mla_attn, with the split scratch in the library's fixed
    device array instead of a workspace (see dsa_sparse_mla_attn_static)."""
    if out is None:
        out = torch.empty(shape.batch, shape.n_q, shape.heads, shape.d_v, dtype=q.dtype, device=q.device)
    _check(lib().dsa_sparse_mla_attn_static(ctypes.byref(shape), _p(q), _p(kv), _p(v), _p(idx), _p(ctx_len),
                                            _p(out), _p(lse), _stream(stream)), "dsa_sparse_mla_attn_static")
    return out


def hadamard_quant_fp8(x, x8=None, scale=None, stream=None):
    """Rotate + quantise rows of 128: returns (codes uint8, scale fp32)."""
    dim = x.shape[-1]
    rows = x.numel() // dim
    if x8 is None:
        x8 = torch.empty(x.shape, dtype=torch.uint8, device=x.device)
    if scale is None:
        scale = torch.empty(x.shape[:-1], dtype=torch.float32, device=x.device)
    _check(lib().dsa_hadamard_quant_fp8(_p(x), _dtype_code(x.dtype), rows, dim, _p(x8), _p(scale),
                                        _stream(stream)), "dsa_hadamard_quant_fp8")
    return x8, scale


def cache_append(shape, k_new, kv_new, pos, k_cache, kv_cache, k_scale=None, v_new=None, v_cache=None,
                 stream=None):
    """Write new tokens into the caches at rows pos[b] + i (see dsa_cache_append).

    k_new [B, n_new, idx_dim], kv_new [B, n_new, ...]; with idx_dtype E4M3 the
    keys are rotated + quantised into k_cache (uint8) and k_scale."""
    n_new = k_new.shape[1] if k_new.dim() > 1 else 0
    _check(lib().dsa_cache_append(ctypes.byref(shape), n_new, _p(k_new), _p(kv_new), _p(v_new), _p(pos),
                                  _p(k_cache), _p(k_scale), _p(kv_cache), _p(v_cache), _stream(stream)),
           "dsa_cache_append")


def forward(shape, q_idx, k_idx, w, q, kv, ctx_len, q_pos0, out=None, v=None, q_scale=None, k_scale=None,
            lse=None, idx_out=None, workspace=None, stream=None, k_rescore=None):
    """The whole layer step (see dsa_forward); returns out."""
    if out is None:
        out = torch.empty(shape.batch, shape.n_q, shape.heads, shape.d_v, dtype=q.dtype, device=q.device)
    ws, n = _workspace(shape, WS_FORWARD, workspace, q.device)
    _check(lib().dsa_forward(ctypes.byref(shape), _p(q_idx), _p(q_scale), _p(k_idx), _p(k_scale), _p(k_rescore),
                             _p(w), _p(q),
                             _p(kv), _p(v), _p(ctx_len), _p(q_pos0), _p(out), _p(lse), _p(idx_out), _p(ws), n,
                             _stream(stream)), "dsa_forward")
    return out


def forward_host(shape, h_q_idx, h_w, h_q, h_ctx_len, h_q_pos0, k_idx, kv, h_out, v=None, k_scale=None,
                 h_lse=None, workspace=None, stream=None, k_rescore=None):
    """The layer step with this step's tensors in host memory (see dsa_forward_host)."""
    ws, n = _workspace(shape, WS_FORWARD_HOST, workspace, k_idx.device)
    _check(lib().dsa_forward_host(ctypes.byref(shape), _p(h_q_idx), _p(h_w), _p(h_q), _p(h_ctx_len), _p(h_q_pos0),
                                  _p(k_idx), _p(k_scale), _p(k_rescore), _p(kv), _p(v), _p(h_out), _p(h_lse), _p(ws), n,
                                  _stream(stream)), "dsa_forward_host")
    return h_out


def forward_host_async(shape, h_q_idx, h_w, h_q, h_ctx_len, h_q_pos0, k_idx, kv, h_out, done=None, v=None,
                       k_scale=None, h_lse=None, workspace=None, stream=None, k_rescore=None):
    """The host-buffer step, returning once enqueued (see dsa_forward_host_async).
    `done`: a torch.cuda.Event recorded once h_out / h_lse hold this call's
    outputs (or None)."""
    ws, n = _workspace(shape, WS_FORWARD_HOST, workspace, k_idx.device)
    ev = None
    if done is not None:
        if not done.cuda_event:  # torch creates the event on its first record
            done.record(torch.cuda.current_stream(k_idx.device))
        ev = done.cuda_event
    _check(lib().dsa_forward_host_async(ctypes.byref(shape), _p(h_q_idx), _p(h_w), _p(h_q), _p(h_ctx_len),
                                        _p(h_q_pos0), _p(k_idx), _p(k_scale), _p(k_rescore), _p(kv), _p(v), _p(h_out), _p(h_lse),
                                        _p(ws), n, ev, _stream(stream)), "dsa_forward_host_async")
    return h_out


def selftest_wait_timeout(stream=None):
    """Enqueue the bounded-wait diagnostic (see dsa_selftest_wait_timeout)."""
    _check(lib().dsa_selftest_wait_timeout(_stream(stream)), "dsa_selftest_wait_timeout")


def get_error(clear=True):
    """(status, raw word) of the device error word; synchronises the device."""
    word = ctypes.c_uint32(0)
    rc = lib().dsa_get_error(1 if clear else 0, ctypes.byref(word))
    return rc, word.value
