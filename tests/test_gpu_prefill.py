"""GPU parity at the full prefill shapes the benchmark times (DeepSeek-V3.2
configuration: 64 index heads x 128, index_topk 2048, 128 MLA heads over the
576-wide latent).  The step runs as the benchmark runs it -- dsa_forward in
rounds of 4096 queries -- and the fp64 oracle checks:

  * prefill8k (L = 8192): indexer scores and top-k sets of every row, and the
    attention output of 512 rows drawn uniformly (numpy PCG64, seed 1) plus
    rows {0, 2047, 2048, 8191};
  * prefill64k (L = 65536): scores, top-k sets and outputs of 512 rows drawn
    the same way plus rows {0, 2047, 2048, 65535}.

Tolerances are those of the other parity tests (tests/_parity.py).
"""
import numpy as np
import pytest
import torch

import long_context_indexing_lightning_b200 as dsa
import oracle
import workloads
from long_context_indexing_lightning_b200 import build

from _parity import ATTN_ATOL_BF16, check_idx_valid, check_scores, check_topk_near_ties

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

DEV = "cuda"
CHUNK = 4096
H = workloads.to_numpy


@pytest.fixture(scope="module", autouse=True)
def _setup():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build.build()
    dsa.lib()
    dsa.get_error(clear=True)
    yield
    rc, word = dsa.get_error(clear=True)
    assert rc == 0, f"device error word {word:#x} after the module"


def _scores_of_rows(shape, t, picks):
    """GPU indexer scores of the picked query rows, computed in rounds of
    CHUNK queries (as the step computes them)."""
    L = shape.n_q
    ld = (shape.s_max + 3) // 4 * 4
    out = np.empty((len(picks), shape.s_max), dtype=np.float32)
    picks = np.asarray(picks)
    buf = torch.empty(1, CHUNK, ld, dtype=torch.float32, device=DEV)
    for r0 in range(0, L, CHUNK):
        c = min(CHUNK, L - r0)
        sel = np.nonzero((picks >= r0) & (picks < r0 + c))[0]
        if sel.size == 0:
            continue
        sh = shape.replace(n_q=c)
        sc = dsa.indexer_scores(sh, t["q_idx"][:, r0:r0 + c], t["k_idx"], t["w"][:, r0:r0 + c], t["ctx_len"],
                                t["q_pos0"] + r0, scores=buf[:, :c])
        rows = torch.from_numpy(picks[sel] - r0).to(DEV)
        out[sel] = sc[0].index_select(0, rows)[:, :shape.s_max].cpu().numpy()
    return out


def _run(name, score_rows, attn_rows):
    wl = workloads.get(name)
    t = workloads.make_inputs(wl, DEV, seed=0)
    shape = dsa.shape_from_workload(wl, q_chunk=CHUNK)
    idx_out = torch.empty(1, wl.n_q, wl.topk, dtype=torch.int32, device=DEV)
    out = dsa.forward(shape, t["q_idx"], t["k_idx"], t["w"], t["q"], t["kv"], t["ctx_len"], t["q_pos0"],
                      idx_out=idx_out)
    torch.cuda.synchronize()
    assert dsa.get_error()[0] == 0

    h = {k: H(t[k]) for k in ("q_idx", "k_idx", "w", "ctx_len", "q_pos0")}
    # indexer scores and top-k sets
    g_sc = _scores_of_rows(dsa.shape_from_workload(wl), t, score_rows)
    rows = [(0, r) for r in score_rows]
    o_sc = oracle.indexer_scores(h["q_idx"], h["k_idx"], h["w"], h["ctx_len"], h["q_pos0"], rows=rows)
    check_scores(g_sc, o_sc, [wl.s_max] * len(rows))
    pos = np.asarray(score_rows, dtype=np.int32)
    o_idx = oracle.topk(np.where(np.isfinite(o_sc), o_sc, -np.inf).astype(np.float32), pos, wl.topk)
    g_idx = idx_out[0].index_select(0, torch.from_numpy(pos.astype(np.int64)).to(DEV)).cpu().numpy()
    check_idx_valid(g_idx, pos, wl.topk)
    check_topk_near_ties(g_idx, o_idx, o_sc, wl.topk)

    # attention outputs on the oracle's selection (positions are in idx:
    # the queries of the checked rows can be passed on their own)
    where = {r: i for i, r in enumerate(score_rows)}
    sel = np.asarray(attn_rows, dtype=np.int64)
    q_sub = H(t["q"][:, torch.from_numpy(sel).to(DEV)])
    o = oracle.sparse_attn(q_sub, H(t["kv"]), o_idx[[where[r] for r in attn_rows]], wl.sm_scale, v=wl.d_v,
                           rows=[(0, i) for i in range(sel.size)])
    got = out[0].index_select(0, torch.from_numpy(sel).to(DEV)).float().cpu().numpy().astype(np.float64)
    err = np.abs(got - o).max()
    assert err <= ATTN_ATOL_BF16, err


def test_forward_prefill8k_all_rows_selected_sampled_outputs():
    L = 8192
    sample = workloads.sample_rows(L, 512, seed=1, extra=(0, 2047, 2048, L - 1))
    _run("prefill8k", list(range(L)), sample)


def test_forward_prefill64k_sampled_rows():
    L = 65536
    sample = workloads.sample_rows(L, 512, seed=1, extra=(0, 2047, 2048, L - 1))
    _run("prefill64k", sample, sample)
