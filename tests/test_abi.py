"""The C ABI library without a GPU: it builds for sm_100a, loads, exports
every function include/dsa.h declares, and its host-side checks and
workspace arithmetic behave (no compute calls)."""
import ctypes
import os
import re

import pytest

import long_context_indexing_lightning_b200 as dsa
from long_context_indexing_lightning_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    build.build()
    return dsa.lib()


def _declared():
    txt = open(os.path.join(ROOT, "include", "dsa.h")).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return sorted(set(re.findall(r"\b(dsa_[a-z0-9_]+)\s*\(", txt)))


def test_every_declared_symbol_is_exported(L):
    names = _declared()
    assert len(names) >= 10
    for n in names:
        assert hasattr(L, n), n
    assert set(names) == set(dsa.EXPORTS)


def test_shape_struct_matches_header():
    txt = open(os.path.join(ROOT, "include", "dsa.h")).read()
    body = txt[txt.index("typedef struct {"):txt.index("} dsa_shape_t;")]
    fields = re.findall(r"\b(?:int32_t|float)\s+([a-z_0-9, ]+);", body)
    names = [f.strip() for group in fields for f in group.split(",")]
    assert names == [f[0] for f in dsa.Shape._fields_]
    assert ctypes.sizeof(dsa.Shape) == 4 * len(names)


def test_status_strings_and_version(L):
    for code in range(7):
        assert L.dsa_status_string(code)
    assert L.dsa_version() >= 100


def test_argument_errors_need_no_gpu(L):
    s = dsa.make_shape(2, 1, 1024)
    # null shape / null pointers are rejected before any CUDA call
    assert L.dsa_indexer_scores(None, None, None, None, None, None, None, None, None, 1024, None) == 1
    assert L.dsa_indexer_scores(ctypes.byref(s), None, None, None, None, None, None, None, None, 1024, None) == 1
    assert L.dsa_topk(ctypes.byref(s), None, 1024, None, None, None, None, 0, None) == 1
    bad = s.replace(idx_scale=0.0)
    assert L.dsa_indexer_scores(ctypes.byref(bad), 16, None, 16, None, 16, 16, 16, 16, 1024, None) == 1
    bad = s.replace(heads=6, kv_heads=4)
    assert L.dsa_workspace_bytes(ctypes.byref(bad), dsa.WS_FORWARD) == 0
    # misaligned score pointer / bad leading dimension
    assert L.dsa_topk(ctypes.byref(s), 18, 1024, 16, 16, 16, None, 0, None) == 1
    assert L.dsa_topk(ctypes.byref(s), 16, 1022, 16, 16, 16, None, 0, None) == 1
    # unsupported tensor-core shapes are reported as such
    odd = s.replace(idx_dim=96)
    assert L.dsa_indexer_scores(ctypes.byref(odd), 16, None, 16, None, 16, 16, 16, 16, 1024, None) == 2
    assert L.dsa_hadamard_quant_fp8(16, dsa.DSA_BF16, 4, 64, 16, 16, None) == 2
    # cache append: null buffers, one-sided v, missing FP8 scales, odd rows
    assert L.dsa_cache_append(ctypes.byref(s), 1, None, 16, None, 16, 16, None, 16, None, None) == 1
    assert L.dsa_cache_append(ctypes.byref(s), -1, 16, 16, None, 16, 16, None, 16, None, None) == 1
    assert L.dsa_cache_append(ctypes.byref(s), 1, 16, 16, 16, 16, 16, None, 16, None, None) == 1
    e4 = s.replace(idx_dtype=dsa.DSA_E4M3)
    assert L.dsa_cache_append(ctypes.byref(e4), 1, 16, 16, None, 16, 16, None, 16, None, None) == 1
    assert L.dsa_cache_append(ctypes.byref(e4.replace(idx_dim=64)), 1, 16, 16, None, 16, 16, 16, 16, None, None) == 2
    assert L.dsa_cache_append(ctypes.byref(s.replace(d_qk=575)), 1, 16, 16, None, 16, 16, None, 16, None, None) == 2
    assert L.dsa_cache_append(ctypes.byref(s), 1, 18, 16, None, 16, 16, None, 16, None, None) == 1
    # host-buffer step, asynchronous form: null inputs, a workspace too small
    assert L.dsa_forward_host_async(ctypes.byref(s), None, None, None, None, None, 16, None, None, 16, None, 16,
                                    None, 16, 1 << 30, None, None) == 1
    assert L.dsa_forward_host_async(ctypes.byref(s), 16, 16, 16, 16, 16, 16, None, None, 16, None, 16, None,
                                    16, 16, None, None) == 3
    # e4m3 step with re-scoring: the bf16 key cache is required, and only then
    e4r = e4.replace(idx_rescore=1024)
    assert L.dsa_forward(ctypes.byref(e4r), 16, None, 16, 16, None, 16, 16, 16, None, 16, 16, 16, None, None,
                         16, 1 << 30, None) == 1
    assert L.dsa_forward(ctypes.byref(s), 16, None, 16, None, 16, 16, 16, 16, None, 16, 16, 16, None, None,
                         16, 1 << 30, None) == 1
    assert L.dsa_forward(ctypes.byref(s.replace(idx_rescore=-1)), 16, None, 16, None, None, 16, 16, 16, None, 16,
                         16, 16, None, None, 16, 1 << 30, None) == 1
    # re-scoring and candidate selection: null lists, lists shorter than n_cand
    assert L.dsa_indexer_rescore(ctypes.byref(s), 16, 16, 16, None, 1024, 1024, 16, 16, 16, 1024, None) == 1
    assert L.dsa_indexer_rescore(ctypes.byref(s), 16, 16, 16, 16, 1000, 1024, 16, 16, 16, 1024, None) == 1
    assert L.dsa_indexer_rescore(ctypes.byref(s.replace(idx_heads=48)), 16, 16, 16, 16, 1024, 1024, 16, 16, 16,
                                 1024, None) == 2
    assert L.dsa_topk_candidates(ctypes.byref(s), 16, None, 1024, 1024, 16, 16, 16, None) == 1
    assert L.dsa_topk_candidates(ctypes.byref(s), 16, 16, 1022, 1022, 16, 16, 16, None) == 1


def test_workspace_arithmetic(L):
    s = dsa.make_shape(32, 1, 131072)
    fwd = dsa.workspace_bytes(s, dsa.WS_FORWARD)
    # scores of the whole batch (fp32) + indices must fit
    assert fwd >= 32 * 131072 * 4 + 32 * 2048 * 4
    host = dsa.workspace_bytes(s, dsa.WS_FORWARD_HOST)
    assert host > fwd
    # chunked prefill bounds the score buffer by the chunk
    p = dsa.make_shape(1, 65536, 65536, q_chunk=4096)
    assert dsa.workspace_bytes(p, dsa.WS_FORWARD) < 4096 * 65536 * 4 * 1.2
    full = p.replace(q_chunk=0)
    assert dsa.workspace_bytes(full, dsa.WS_FORWARD) >= 65536 * 65536 * 4
    # e4m3 with re-scoring adds the candidate lists and their bf16 scores
    e4 = s.replace(idx_dtype=dsa.DSA_E4M3)
    e4r = e4.replace(idx_rescore=1024)
    assert dsa.workspace_bytes(e4r, dsa.WS_FORWARD) >= dsa.workspace_bytes(e4, dsa.WS_FORWARD) + 2 * 32 * 3072 * 4
