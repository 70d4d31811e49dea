"""The allocation-free attention entry point (dsa_sparse_mla_attn_static).

It serves callers that cannot give the library device memory on their
decode path; it must produce what dsa_sparse_mla_attn produces with a
caller-provided workspace.  This file is collected last so that a run which
stops at the first failure has run every other test before it.
"""
import ctypes

import numpy as np
import pytest
import torch

import long_context_indexing_lightning_b200 as dsa
import workloads
from long_context_indexing_lightning_b200 import build

pytestmark = pytest.mark.gpu


def _case(wl, seed):
    t = workloads.make_inputs(wl, "cuda", seed=seed)
    g = np.random.default_rng(seed)
    idx = np.full((wl.batch, wl.topk), -1, dtype=np.int32)
    for b, L in enumerate(wl.lengths()):
        n = min(wl.topk, L)
        idx[b, :n] = np.sort(g.choice(L, size=n, replace=False))
    return t, torch.from_numpy(idx).cuda().reshape(wl.batch, 1, wl.topk)


@pytest.mark.parametrize("name,overrides", [
    ("decode32k", dict(batch=8, s_max=8192)),                        # several splits per query
    ("decode32k", dict(batch=1, s_max=4096)),                        # the most splits: one query
    ("decode32k", dict(batch=32, s_max=4096, ctx_len=tuple([4096] * 31 + [100]))),
])
def test_static_scratch_matches_workspace_entry_point(name, overrides):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build.build()
    L = dsa.lib()
    wl = workloads.get(name, **overrides)
    shape = dsa.shape_from_workload(wl)
    for call, seed in enumerate((21, 22)):      # two calls in a row, different inputs
        t, idx = _case(wl, seed)
        lse_ref = torch.empty(wl.batch, 1, wl.heads, dtype=torch.float32, device="cuda")
        ref = dsa.sparse_mla_attn(shape, t["q"], t["kv"], idx, t["ctx_len"], lse=lse_ref)
        out = torch.full_like(ref, float("nan"))
        lse = torch.full_like(lse_ref, float("nan"))
        stream = torch.cuda.current_stream().cuda_stream
        torch.cuda.synchronize()
        free_before = torch.cuda.mem_get_info()[0]
        rc = L.dsa_sparse_mla_attn_static(ctypes.byref(shape), t["q"].data_ptr(), t["kv"].data_ptr(), None,
                                          idx.data_ptr(), t["ctx_len"].data_ptr(), out.data_ptr(),
                                          lse.data_ptr(), stream)
        assert rc == 0, dsa.STATUS.get(rc, rc)
        torch.cuda.synchronize()
        if call > 0:
            # after the first call (which may load the module and place the
            # array), a call takes no device memory
            assert torch.cuda.mem_get_info()[0] == free_before
        # the same kernels with the same split plan as the workspace call:
        # identical results, bit for bit
        torch.testing.assert_close(out, ref, rtol=0, atol=0)
        torch.testing.assert_close(lse, lse_ref, rtol=0, atol=0)
    rc, word = dsa.get_error(clear=True)
    assert rc == 0, f"device error word {word:#x}"
