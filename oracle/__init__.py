"""Plain fp64 CPU oracle for the DSA layer step -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline
leg may import this package.  It shares no code with the CUDA library and
never imports it.  Arrays are numpy; bf16 data is passed as its uint16 bit
patterns (``torch.Tensor.view(torch.int16)`` on the caller's side) and fp8
data as uint8 e4m3 codes.  The arithmetic lives in ``dsa_oracle.c``; this
module only marshals arguments.

Each function cites the passage of the DeepSeek-V3.2 model documentation
page (Transformers) that it follows -- see the C source for the full text.
"""
import ctypes
import os

import numpy as np

from . import build as _build

F32, BF16, E4M3 = 0, 1, 2

_lib = None


def _load():
    global _lib
    if _lib is None:
        path = _build.build()
        lib = ctypes.CDLL(path)
        P = ctypes.c_void_p
        i32, i64, f64 = ctypes.c_int, ctypes.c_int64, ctypes.c_double
        lib.orc_indexer_scores.argtypes = [i32, i32, i32, i32, P, i32, P, i32, P, P, P, f64, i32, P, P, P]
        lib.orc_indexer_scores_fp8.argtypes = [i32, i32, i32, i32, P, P, P, P, P, P, P, f64, i32, P, P, P]
        lib.orc_hadamard.argtypes = [i32, i64, P, P]
        lib.orc_hadamard_quant_rows.argtypes = [i32, i64, P, i32, P, P, P]
        lib.orc_e4m3_encode.argtypes = [f64]
        lib.orc_e4m3_encode.restype = ctypes.c_uint8
        lib.orc_e4m3_decode.argtypes = [ctypes.c_uint8]
        lib.orc_e4m3_decode.restype = f64
        lib.orc_e4m3_encode_array.argtypes = [i64, P, P]
        lib.orc_e4m3_decode_array.argtypes = [i64, P, P]
        lib.orc_topk.argtypes = [i32, i64, P, P, i32, P]
        lib.orc_topk.restype = i32
        lib.orc_sparse_attn.argtypes = [i32, i32, i32, i32, i32, i32, P, i32, P, i32, P, i32,
                                        P, i32, f64, i32, P, P, P, P]
        lib.orc_dense_masked_attn.argtypes = [i32, i32, i32, i32, i32, i32, P, i32, P, i32, P, i32,
                                              P, P, i32, f64, i32, P, P, P]
        lib.orc_linear.argtypes = [i64, i32, i32, P, i32, P, i32, P]
        lib.orc_num_threads.restype = i32
        _lib = lib
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _typed(a):
    """(contiguous array, dtype code) for fp32 / bf16-bits / e4m3-code arrays."""
    a = np.ascontiguousarray(a)
    if a.dtype == np.float32:
        return a, F32
    if a.dtype in (np.uint16, np.int16):
        return a.view(np.uint16), BF16
    if a.dtype == np.uint8:
        return a, E4M3
    if a.dtype == np.float64:
        raise TypeError("oracle inputs are stored types (fp32, bf16 bits, e4m3 codes), not fp64")
    raise TypeError(f"unsupported oracle input dtype {a.dtype}")


def _rows(rows, B, n_q):
    if rows is None:
        bb, tt = np.meshgrid(np.arange(B, dtype=np.int32), np.arange(n_q, dtype=np.int32), indexing="ij")
        return bb.reshape(-1).copy(), tt.reshape(-1).copy()
    rows = np.asarray(rows, dtype=np.int32).reshape(-1, 2)
    return np.ascontiguousarray(rows[:, 0]), np.ascontiguousarray(rows[:, 1])


def num_threads() -> int:
    return int(_load().orc_num_threads())


def indexer_scores(q, k, w, ctx_len, q_pos0, scale=1.0, rows=None):
    """Lightning-indexer scores (DeepSeek-V3.2 doc, section DSA, item 1).

    q [B, n_q, H, D], k [B, s_max, D] (fp32 or bf16 bits), w [B, n_q, H] fp32.
    Returns fp64 [nrows, s_max]: the ReLU-weighted head sum for s <= pos,
    -inf for pos < s < ctx_len, NaN for s >= ctx_len.
    """
    B, n_q, H, D = q.shape
    s_max = k.shape[1]
    q, qt = _typed(q)
    k, kt = _typed(k)
    w = np.ascontiguousarray(w, dtype=np.float32)
    ctx = np.ascontiguousarray(ctx_len, dtype=np.int32)
    pos0 = np.ascontiguousarray(q_pos0, dtype=np.int32)
    rb, rt = _rows(rows, B, n_q)
    out = np.empty((rb.size, s_max), dtype=np.float64)
    _load().orc_indexer_scores(n_q, s_max, H, D, _ptr(q), qt, _ptr(k), kt, _ptr(w), _ptr(ctx), _ptr(pos0),
                               float(scale), rb.size, _ptr(rb), _ptr(rt), _ptr(out))
    return out


def indexer_scores_fp8(q_code, q_sigma, k_code, k_sigma, w, ctx_len, q_pos0, scale=1.0, rows=None):
    """FP8 indexer scores on e4m3 codes and per-row scales (section DSA, item 1)."""
    B, n_q, H, D = q_code.shape
    s_max = k_code.shape[1]
    qc = np.ascontiguousarray(q_code, dtype=np.uint8)
    kc = np.ascontiguousarray(k_code, dtype=np.uint8)
    qs = np.ascontiguousarray(q_sigma, dtype=np.float32)
    ks = np.ascontiguousarray(k_sigma, dtype=np.float32)
    w = np.ascontiguousarray(w, dtype=np.float32)
    ctx = np.ascontiguousarray(ctx_len, dtype=np.int32)
    pos0 = np.ascontiguousarray(q_pos0, dtype=np.int32)
    rb, rt = _rows(rows, B, n_q)
    out = np.empty((rb.size, s_max), dtype=np.float64)
    _load().orc_indexer_scores_fp8(n_q, s_max, H, D, _ptr(qc), _ptr(qs), _ptr(kc), _ptr(ks), _ptr(w),
                                   _ptr(ctx), _ptr(pos0), float(scale), rb.size, _ptr(rb), _ptr(rt), _ptr(out))
    return out


def hadamard(x):
    """Orthonormal Sylvester-Hadamard rotation of each last-axis vector (fp64)."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    n = x.shape[-1]
    y = np.empty_like(x)
    _load().orc_hadamard(n, x.size // n, _ptr(x), _ptr(y))
    return y


def hadamard_quant(x):
    """Rotate rows by H, scale by amax/448, code as e4m3.

    Returns (codes uint8 [..., n], sigma fp32 [...], quotient fp64 [..., n]).
    """
    xa, xt = _typed(x)
    n = xa.shape[-1]
    rows = xa.size // n
    code = np.empty(xa.shape, dtype=np.uint8)
    sigma = np.empty(xa.shape[:-1], dtype=np.float32)
    quot = np.empty(xa.shape, dtype=np.float64)
    _load().orc_hadamard_quant_rows(n, rows, _ptr(xa), xt, _ptr(code), _ptr(sigma), _ptr(quot))
    return code, sigma, quot


def cache_append(k_cache, kv_cache, k_new, kv_new, pos, k_scale=None, v_cache=None, v_new=None):
    """Cache append (section DSA: the indexer keeps its own per-token key
    cache, single head, beside the K/V cache, updated through
    update_indexer(); the reference indexer runs in FP8 after the Hadamard
    rotation, item 1).

    New token i of sequence b lands in cache row pos[b] + i; rows outside
    [0, s_max) are skipped.  k_cache in a stored type (fp32, bf16 bits) gets
    the key copied; a uint8 (e4m3) k_cache gets the rotated, quantised codes
    and k_scale the row scale, as hadamard_quant computes them.  kv / v rows
    are copied.  Returns updated copies (k_cache, k_scale, kv_cache, v_cache).
    """
    k_cache = np.array(k_cache, copy=True)
    kv_cache = np.array(kv_cache, copy=True)
    k_scale = None if k_scale is None else np.array(k_scale, copy=True)
    v_cache = None if v_cache is None else np.array(v_cache, copy=True)
    fp8 = k_cache.dtype == np.uint8
    if fp8:
        codes, sigma, _ = hadamard_quant(k_new)
    B, n = k_new.shape[0], k_new.shape[1]
    s_max = k_cache.shape[1]
    for b in range(B):
        for i in range(n):
            r = int(pos[b]) + i
            if r < 0 or r >= s_max:
                continue
            if fp8:
                k_cache[b, r] = codes[b, i]
                k_scale[b, r] = sigma[b, i]
            else:
                k_cache[b, r] = k_new[b, i]
            kv_cache[b, r] = kv_new[b, i]
            if v_cache is not None:
                v_cache[b, r] = v_new[b, i]
    return k_cache, k_scale, kv_cache, v_cache


def linear(x, w):
    """The indexer's projections (DeepSeek-V3.2 doc: `wq_b` on the query
    latent, the single-head key projection, `weights_proj`): Y = X W^T in fp64.

    x [..., K] and w [N, K] in a stored type (fp32 or bf16 bits).  Returns
    fp64 [..., N].
    """
    xa, xt = _typed(x)
    wa, wt = _typed(w)
    K = xa.shape[-1]
    N = wa.shape[0]
    if wa.shape[1] != K:
        raise ValueError("x and w disagree on K")
    M = xa.size // K
    y = np.empty(xa.shape[:-1] + (N,), dtype=np.float64)
    _load().orc_linear(M, N, K, _ptr(xa), xt, _ptr(wa), wt, _ptr(y))
    return y


def e4m3_encode(x):
    x = np.ascontiguousarray(x, dtype=np.float64)
    out = np.empty(x.shape, dtype=np.uint8)
    _load().orc_e4m3_encode_array(x.size, _ptr(x), _ptr(out))
    return out


def e4m3_decode(c):
    c = np.ascontiguousarray(c, dtype=np.uint8)
    out = np.empty(c.shape, dtype=np.float64)
    _load().orc_e4m3_decode_array(c.size, _ptr(c), _ptr(out))
    return out


def topk(scores, pos, k):
    """Top-k selection (section DSA, item 2).

    scores fp32 [nrows, >= max(pos)+1], pos int [nrows] (the query position
    of each row).  Returns int32 [nrows, k]: the kept indices ascending,
    padded with -1.
    """
    scores = np.ascontiguousarray(scores, dtype=np.float32)
    pos = np.ascontiguousarray(pos, dtype=np.int32)
    nrows, ld = scores.shape
    if pos.size and int(pos.max()) >= ld:
        raise ValueError("row shorter than its query position")
    idx = np.empty((nrows, k), dtype=np.int32)
    bad = _load().orc_topk(nrows, ld, _ptr(scores), _ptr(pos), int(k), _ptr(idx))
    if bad:
        raise ValueError(f"{bad} non-finite candidate scores")
    return idx


def sparse_attn(q, kv, idx, sm_scale, v=None, rows=None, want_lse=False):
    """Attention over the selected keys only (section DSA, item 2).

    q [B, n_q, H, d_qk]; kv [B, s_max, KVH, d_qk] (or [B, s_max, d_qk] for the
    single shared latent row); v [B, s_max, KVH, d_v] or None (value = first
    d_v columns of kv, the absorbed MLA form: then d_v must be given through
    ``v=int``).  idx [nrows, k] int32.  Returns fp64 out [nrows, H, d_v]
    (and lse [nrows, H]).
    """
    B, n_q, H, d_qk = q.shape
    if kv.ndim == 3:
        kv = kv.reshape(kv.shape[0], kv.shape[1], 1, kv.shape[2])
    s_max, KVH = kv.shape[1], kv.shape[2]
    if isinstance(v, int):
        d_v, va, vt = v, None, 0
    else:
        if v.ndim == 3:
            v = v.reshape(v.shape[0], v.shape[1], 1, v.shape[2])
        va, vt = _typed(v)
        d_v = va.shape[-1]
    qa, qt = _typed(q)
    ka, kt = _typed(kv)
    rb, rt = _rows(rows, B, n_q)
    idx = np.ascontiguousarray(idx, dtype=np.int32).reshape(rb.size, -1)
    k = idx.shape[1]
    out = np.empty((rb.size, H, d_v), dtype=np.float64)
    lse = np.empty((rb.size, H), dtype=np.float64)
    _load().orc_sparse_attn(n_q, s_max, H, KVH, d_qk, d_v, _ptr(qa), qt, _ptr(ka), kt, _ptr(va), vt,
                            _ptr(idx), k, float(sm_scale), rb.size, _ptr(rb), _ptr(rt), _ptr(out), _ptr(lse))
    return (out, lse) if want_lse else out


def dense_masked_attn(q, kv, idx, q_pos0, sm_scale, v=None, rows=None):
    """Dense causal attention with an additive -inf mask off the selected set."""
    B, n_q, H, d_qk = q.shape
    if kv.ndim == 3:
        kv = kv.reshape(kv.shape[0], kv.shape[1], 1, kv.shape[2])
    s_max, KVH = kv.shape[1], kv.shape[2]
    if isinstance(v, int):
        d_v, va, vt = v, None, 0
    else:
        if v.ndim == 3:
            v = v.reshape(v.shape[0], v.shape[1], 1, v.shape[2])
        va, vt = _typed(v)
        d_v = va.shape[-1]
    qa, qt = _typed(q)
    ka, kt = _typed(kv)
    pos0 = np.ascontiguousarray(q_pos0, dtype=np.int32)
    rb, rt = _rows(rows, B, n_q)
    idx = np.ascontiguousarray(idx, dtype=np.int32).reshape(rb.size, -1)
    out = np.empty((rb.size, H, d_v), dtype=np.float64)
    _load().orc_dense_masked_attn(n_q, s_max, H, KVH, d_qk, d_v, _ptr(qa), qt, _ptr(ka), kt, _ptr(va), vt,
                                  _ptr(pos0), _ptr(idx), idx.shape[1], float(sm_scale), rb.size,
                                  _ptr(rb), _ptr(rt), _ptr(out))
    return out
