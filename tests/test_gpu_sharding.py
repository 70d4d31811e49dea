"""The prefill split by query rows (sharding.py) on one GPU.

The ranks' row ranges run one after another on the same device, with no
collective (the cache exchange is covered by the gloo tests in
test_sharding.py): the balanced ranges must reproduce the unsplit prefill's
selections exactly (every score is computed the same way whichever rows share
a launch, and the top-k is exact on identical scores) and its outputs within
the attention tolerance (the split-K layout of the attention may differ with
the number of rows), and one rank's append-then-score must equal scoring its
rows on the filled caches.
"""
import numpy as np
import pytest
import torch

import long_context_indexing_lightning_b200 as dsa
import oracle
import workloads
from long_context_indexing_lightning_b200 import build, sharding

from _parity import check_idx_valid, check_topk_near_ties

pytestmark = pytest.mark.gpu

DEV = "cuda"
ATTN_ATOL_BF16 = 2e-2


@pytest.fixture(scope="module", autouse=True)
def _setup():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build.build()
    dsa.lib()
    dsa.get_error(clear=True)
    yield


def _rows(x, r0, r1):
    return x[:, r0:r1].contiguous()


def test_balanced_row_ranges_reproduce_the_unsplit_prefill():
    wl = workloads.get("prefill8k", n_q=1536, s_max=1536, topk=512)
    t = workloads.make_inputs(wl, DEV, seed=31)
    shape = dsa.shape_from_workload(wl)
    idx_full = torch.empty(1, wl.n_q, wl.topk, dtype=torch.int32, device=DEV)
    full = dsa.forward(shape, t["q_idx"], t["k_idx"], t["w"], t["q"], t["kv"], t["ctx_len"], t["q_pos0"],
                       idx_out=idx_full)
    outs, idxs = [], []
    ranges = sharding.balanced_row_ranges(wl.n_q, 3, topk=wl.topk)
    for r0, r1 in ranges:
        idx = torch.empty(1, r1 - r0, wl.topk, dtype=torch.int32, device=DEV)
        outs.append(dsa.forward(sharding.rank_shape(shape, r0, r1), _rows(t["q_idx"], r0, r1), t["k_idx"],
                                _rows(t["w"], r0, r1), _rows(t["q"], r0, r1), t["kv"], t["ctx_len"],
                                t["q_pos0"] + r0, idx_out=idx))
        idxs.append(idx)
    torch.testing.assert_close(torch.cat(idxs, 1), idx_full, rtol=0, atol=0)
    assert (torch.cat(outs, 1).float() - full.float()).abs().max().item() <= ATTN_ATOL_BF16
    assert dsa.get_error()[0] == 0
    # and the split run against the oracle, on rows of every rank's range
    # (each range's first and last row, and one inside)
    H = workloads.to_numpy
    h = {k: H(v) for k, v in t.items()}
    picks = sorted({r for r0, r1 in ranges for r in (r0, (r0 + r1) // 2, r1 - 1)})
    rows = [(0, r) for r in picks]
    o_sc = oracle.indexer_scores(h["q_idx"], h["k_idx"], h["w"], h["ctx_len"], h["q_pos0"], rows=rows)
    pos = np.array(picks, dtype=np.int32)
    o_idx = oracle.topk(np.where(np.isfinite(o_sc), o_sc, -np.inf).astype(np.float32), pos, wl.topk)
    g_idx = torch.cat(idxs, 1)[0, picks].cpu().numpy()
    check_idx_valid(g_idx, pos, wl.topk)
    check_topk_near_ties(g_idx, o_idx, o_sc, wl.topk)
    o = oracle.sparse_attn(h["q"], h["kv"], o_idx, wl.sm_scale, v=wl.d_v, rows=rows)
    got = torch.cat(outs, 1)[0, picks].float().cpu().numpy().astype(np.float64)
    assert np.abs(got - o).max() <= ATTN_ATOL_BF16


def test_prefill_rank_appends_then_scores_its_rows():
    wl = workloads.get("prefill8k", n_q=1024, s_max=1024, topk=256)
    t = workloads.make_inputs(wl, DEV, seed=32)
    shape = dsa.shape_from_workload(wl)
    k_cache = torch.zeros_like(t["k_idx"])
    kv_cache = torch.zeros_like(t["kv"])
    r0, r1 = 200, 700
    got = sharding.prefill_rank(dsa, shape, 0, (r0, r1), t["k_idx"], t["kv"], k_cache, kv_cache,
                                _rows(t["q_idx"], r0, r1), _rows(t["w"], r0, r1), _rows(t["q"], r0, r1),
                                t["ctx_len"])
    torch.testing.assert_close(k_cache, t["k_idx"], rtol=0, atol=0)
    torch.testing.assert_close(kv_cache, t["kv"], rtol=0, atol=0)
    want = dsa.forward(sharding.rank_shape(shape, r0, r1), _rows(t["q_idx"], r0, r1), t["k_idx"],
                       _rows(t["w"], r0, r1), _rows(t["q"], r0, r1), t["kv"], t["ctx_len"], t["q_pos0"] + r0)
    torch.testing.assert_close(got, want, rtol=0, atol=0)
    assert dsa.get_error()[0] == 0
