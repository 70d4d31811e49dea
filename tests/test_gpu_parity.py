"""GPU parity: every step of the CUDA path against the fp64 CPU oracle on the
same seeded inputs, called through the C ABI (ctypes binding).

Inputs come from ``workloads`` (seeded draws); expected values only from
``oracle``.  Where a step consumes another step's result (top-k consumes
scores, attention consumes indices) the test feeds both sides the ORACLE's
result, so each kernel is judged on its own.
"""
import math

import numpy as np
import pytest
import torch

import long_context_indexing_lightning_b200 as dsa
import oracle
import workloads
from long_context_indexing_lightning_b200 import build

from _parity import (ATTN_ATOL_BF16, bf16_bits_to_f64, check_idx_valid, check_scores, check_topk_near_ties,
                     rms_finite)

pytestmark = pytest.mark.gpu

DEV = "cuda"
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


def _rows_all(B, n_q):
    return [(b, t) for b in range(B) for t in range(n_q)]


def _pos(wl_or_pos0, rows):
    pos0 = wl_or_pos0
    return np.array([pos0[b] + t for b, t in rows], dtype=np.int32)


def _custom(name, **kw):
    return workloads.get(name, **kw)


def _gpu_scores(shape, t):
    return dsa.indexer_scores(shape, t["q_idx"], t["k_idx"], t["w"], t["ctx_len"], t["q_pos0"])


def _oracle_scores(t, rows, scale=1.0):
    return oracle.indexer_scores(H(t["q_idx"]), H(t["k_idx"]), H(t["w"]), H(t["ctx_len"]), H(t["q_pos0"]),
                                 scale=scale, rows=rows)


def _scores_for_rows(sc, rows):
    n_q = sc.shape[1]
    flat = sc.reshape(-1, sc.shape[2])
    sel = torch.tensor([b * n_q + t for b, t in rows], device=sc.device, dtype=torch.long)
    return flat.index_select(0, sel).cpu().numpy()


# ----------------------------------------------------------------- indexer --

def test_indexer_tiny_fp32_all_rows():
    wl = workloads.get("tiny")
    t = workloads.make_inputs(wl, DEV, seed=0)
    shape = dsa.shape_from_workload(wl)
    sc = _gpu_scores(shape, t)
    rows = _rows_all(wl.batch, wl.n_q)
    ora = _oracle_scores(t, rows)
    check_scores(_scores_for_rows(sc, rows), ora, [wl.s_max] * len(rows))


@pytest.mark.parametrize("H_I", [64, 16, 32, 128])
def test_indexer_bf16_ragged_prefill(H_I):
    """Two sequences of different lengths, queries in the middle of each,
    s_max not a multiple of the 128-key tile, n_q not a multiple of the
    query block."""
    wl = _custom("prefill8k", batch=2, n_q=150, s_max=600, idx_heads=H_I, ctx_len=(600, 433))
    t = workloads.make_inputs(wl, DEV, seed=1, attention=False)
    t["q_pos0"] = torch.tensor([450, 283], dtype=torch.int32, device=DEV)
    shape = dsa.shape_from_workload(wl)
    sc = _gpu_scores(shape, t)
    rows = _rows_all(2, 150)
    ora = _oracle_scores(t, rows)
    check_scores(_scores_for_rows(sc, rows), ora, [600 if b == 0 else 433 for b, _ in rows])


def test_indexer_bf16_decode32k_all_rows():
    wl = workloads.get("decode32k")
    t = workloads.make_inputs(wl, DEV, seed=0, attention=False)
    sc = _gpu_scores(dsa.shape_from_workload(wl), t)
    rows = _rows_all(wl.batch, 1)
    check_scores(_scores_for_rows(sc, rows), _oracle_scores(t, rows), [wl.s_max] * len(rows))


def test_indexer_bf16_decode_ragged_lengths():
    wl = _custom("decode32k", batch=5, s_max=5000, ctx_len=(5000, 1, 129, 4097, 2048))
    t = workloads.make_inputs(wl, DEV, seed=3, attention=False)
    sc = _gpu_scores(dsa.shape_from_workload(wl), t)
    rows = _rows_all(5, 1)
    check_scores(_scores_for_rows(sc, rows), _oracle_scores(t, rows), list(wl.lengths()))


@pytest.mark.slow
def test_indexer_bf16_prefill8k_sampled_rows():
    wl = workloads.get("prefill8k")
    t = workloads.make_inputs(wl, DEV, seed=0, attention=False)
    sc = _gpu_scores(dsa.shape_from_workload(wl), t)
    rows = [(0, r) for r in workloads.sample_rows(wl.n_q, 12, seed=1, extra=(0, 127, 128, 2047, 2048, 8191))]
    check_scores(_scores_for_rows(sc, rows), _oracle_scores(t, rows), [wl.s_max] * len(rows))


@pytest.mark.slow
def test_indexer_bf16_decode128k_sampled_rows():
    wl = workloads.get("decode128k")
    t = workloads.make_inputs(wl, DEV, seed=0, attention=False)
    sc = _gpu_scores(dsa.shape_from_workload(wl), t)
    rows = [(0, 0), (17, 0), (31, 0)]
    # the oracle reads only the sampled sequences' keys
    sub = {"q_idx": t["q_idx"][[0, 17, 31]], "k_idx": t["k_idx"][[0, 17, 31]], "w": t["w"][[0, 17, 31]],
           "ctx_len": t["ctx_len"][[0, 17, 31]], "q_pos0": t["q_pos0"][[0, 17, 31]]}
    ora = _oracle_scores(sub, [(0, 0), (1, 0), (2, 0)])
    check_scores(_scores_for_rows(sc, rows), ora, [wl.s_max] * 3)


# ------------------------------------------------------------------- top-k --

def _topk_gpu(shape, scores_np, ctx, pos0):
    """Run the GPU top-k on host-made scores [B, n_q, S] (fp32)."""
    B, n_q, S = scores_np.shape
    ld = (S + 3) // 4 * 4
    buf = torch.full((B, n_q, ld), float("nan"), dtype=torch.float32, device=DEV)
    buf[:, :, :S] = torch.from_numpy(scores_np).to(DEV)
    idx = dsa.topk(shape, buf, torch.tensor(ctx, dtype=torch.int32, device=DEV),
                   torch.tensor(pos0, dtype=torch.int32, device=DEV))
    return idx.cpu().numpy().reshape(B * n_q, -1)


def _topk_case(B, n_q, S, k, ctx, pos0, scores_np):
    shape = dsa.make_shape(B, n_q, S, topk=k)
    g = _topk_gpu(shape, scores_np, ctx, pos0)
    rows = _rows_all(B, n_q)
    pos = _pos(pos0, rows)
    o = oracle.topk(scores_np.reshape(B * n_q, S), pos, k)
    np.testing.assert_array_equal(g, o)
    check_idx_valid(g, pos, k)


def test_topk_exact_on_oracle_scores_tiny():
    wl = workloads.get("tiny")
    t = workloads.make_inputs(wl, "cpu", seed=0)
    rows = _rows_all(1, wl.n_q)
    sc = _oracle_scores(t, rows).astype(np.float32).reshape(1, wl.n_q, wl.s_max)
    _topk_case(1, wl.n_q, wl.s_max, wl.topk, [wl.s_max], [0], sc)


def test_topk_exact_on_oracle_scores_decode32k():
    wl = workloads.get("decode32k")
    t = workloads.make_inputs(wl, DEV, seed=0, attention=False)
    rows = _rows_all(wl.batch, 1)
    sc = _oracle_scores(t, rows).astype(np.float32).reshape(wl.batch, 1, wl.s_max)
    _topk_case(wl.batch, 1, wl.s_max, wl.topk, wl.lengths(), wl.positions0(), sc)


@pytest.mark.parametrize("seed", [0, 1])
def test_topk_ties_and_zeros_full_length(seed):
    """Seeded fp32 rows with few distinct values (many exact ties), signed
    zeros, and ragged lengths, at the full 128K context, k = 2048."""
    g = np.random.default_rng(seed)
    B, S, k = 6, 131072, 2048
    sc = (g.integers(-40, 40, size=(B, 1, S)).astype(np.float32) * 0.25)
    sc[0] = 0.0
    sc[1, 0, ::3] = -0.0
    sc[2] = np.float32(1.5)
    sc[3, 0, 5000:] = np.float32(-1e30)
    ctx = [S, S, 3000, S, 2048, 2049]
    pos0 = [c - 1 for c in ctx]
    _topk_case(B, 1, S, k, ctx, pos0, sc)


def _structured_rows(g, B, S):
    """Rows radix select finds hardest (the pages print no score
    distribution): a planted recent window (the last 2048 keys score above
    the rest), every score inside one exponent bucket [1, 2), and equal
    scores; the remaining rows gaussian."""
    sc = g.standard_normal((B, 1, S)).astype(np.float32)
    sc[0, 0, S - 2048:] = 4.0 + g.random(2048).astype(np.float32)
    sc[1, 0] = (1.0 + g.random(S)).astype(np.float32)
    sc[2, 0] = np.float32(0.75)
    return sc


def test_topk_structured_rows_decode128k():
    """Exact against the oracle at the 128K shape on the structured rows."""
    g = np.random.default_rng(11)
    B, S, k = 4, 131072, 2048
    sc = _structured_rows(g, B, S)
    _topk_case(B, 1, S, k, [S] * B, [S - 1] * B, sc)


def test_topk_prefill_rows_all_positions():
    """Every query position of a short prefill, including rows with fewer
    than k candidates and rows around the 2048 boundary."""
    g = np.random.default_rng(5)
    n_q, S, k = 2304, 2304, 2048
    sc = g.standard_normal((1, n_q, S)).astype(np.float32)
    sc[0, :, ::7] = np.round(sc[0, :, ::7])       # ties
    _topk_case(1, n_q, S, k, [S], [0], sc)


def test_topk_many_long_rows_walked_in_chunks():
    """A launch with more rows than twice the SM count (a prefill round) runs
    one CTA per row, walking it in 8K-key chunks: 400 query rows at
    positions 39600..39999 of a 40,000-key row (five chunks), gaussian rows
    with exact ties, rows of equal scores and rows inside one exponent bucket
    (the overflow path), exact against the oracle."""
    g = np.random.default_rng(21)
    n_q, S, k = 400, 40000, 2048
    sc = g.standard_normal((1, n_q, S)).astype(np.float32)
    sc[0, :, ::5] = np.round(sc[0, :, ::5] * 4) / 4          # exact ties
    sc[0, 7] = np.float32(-0.5)                              # all equal
    sc[0, 8] = (1.0 + g.random(S)).astype(np.float32)        # one exponent bucket
    sc[0, 9, ::2] = -0.0                                     # signed zeros
    _topk_case(1, n_q, S, k, [S], [S - n_q], sc)


@pytest.mark.parametrize("B,n_q,S", [
    (1, 600, 65536),   # a prefill round: one CTA a row, eight 8K-key chunks, lists overflow
    (24, 1, 131072),   # decode rows: a cluster of four CTAs a row, every list thousands long
])
def test_topk_every_row_with_huge_candidate_bins(B, n_q, S):
    """Every row's candidate bin (the first 11 key bits) holds a quarter of
    the row: scores inside [1, 2) on a grid of 2^-12 (thousands of exact
    ties), a few rows of one value.  One CTA walking a 64K row cannot list
    them (the overflow path); a CTA of a cluster lists its whole slice.
    Exact against the oracle."""
    g = np.random.default_rng(31)
    sc = (1.0 + g.integers(0, 4096, size=(B, n_q, S)) / 4096.0).astype(np.float32)
    sc[0, 0] = np.float32(1.25)
    sc[-1, -1] = np.float32(1.5)
    k = 2048
    if n_q > 1:
        _topk_case(B, n_q, S, k, [S] * B, [S - n_q] * B, sc)
    else:
        _topk_case(B, n_q, S, k, [S] * B, [S - 1] * B, sc)


def test_topk_gaussian_decode128k_shape():
    g = np.random.default_rng(9)
    B, S, k = 32, 131072, 2048
    sc = g.standard_normal((B, 1, S)).astype(np.float32)
    _topk_case(B, 1, S, k, [S] * B, [S - 1] * B, sc)


def _hist_pair(shape, t):
    hist = torch.empty(dsa.workspace_bytes(shape, dsa.WS_HIST), dtype=torch.uint8, device=DEV)
    sc = dsa.indexer_scores_hist(shape, t["q_idx"], t["k_idx"], t["w"], t["ctx_len"], t["q_pos0"], hist)
    got = dsa.topk_hist(shape, sc, t["ctx_len"], t["q_pos0"], hist)
    want = dsa.topk(shape, sc, t["ctx_len"], t["q_pos0"])
    return sc, got, want


@pytest.mark.parametrize("lengths", [
    (131072,) * 8,                               # runs of key tiles spanning two rows
    (131072, 7, 5000, 131072, 40000, 1, 131072, 2049, 90001, 131072),  # ragged, short rows
])
def test_indexer_topk_handoff_equals_plain_topk(lengths):
    """The indexer's first-digit histograms (decode schedule) handed to the
    top-k: the selection is bit-identical to the plain top-k on the same
    scores, and the scores to the plain indexer's."""
    B = len(lengths)
    wl = _custom("decode128k", batch=B, ctx_len=lengths)
    t = workloads.make_inputs(wl, DEV, seed=15, attention=False)
    shape = dsa.shape_from_workload(wl)
    sc, got, want = _hist_pair(shape, t)
    torch.testing.assert_close(got, want, rtol=0, atol=0)
    plain = _gpu_scores(shape, t)
    for b, L in enumerate(lengths):
        torch.testing.assert_close(sc[b, :, :L], plain[b, :, :L], rtol=0, atol=0)
    assert dsa.get_error()[0] == 0


def test_topk_hist_from_another_call_is_reported():
    """Histograms written by one indexer call handed to a top-k over another
    call's scores: the top-k's own count checks flag DSA_ERR_HIST_MISMATCH
    (bounds-checked: nothing outside the buffers is touched), and the next
    matched pair is exact again."""
    wl = workloads.get("decode32k")
    shape = dsa.shape_from_workload(wl)
    ta = workloads.make_inputs(wl, DEV, seed=17, attention=False)
    tb = workloads.make_inputs(wl, DEV, seed=18, attention=False)
    hist = torch.empty(dsa.workspace_bytes(shape, dsa.WS_HIST), dtype=torch.uint8, device=DEV)
    dsa.indexer_scores_hist(shape, ta["q_idx"], ta["k_idx"], ta["w"], ta["ctx_len"], ta["q_pos0"], hist)
    sc_b = _gpu_scores(shape, tb)
    dsa.topk_hist(shape, sc_b, tb["ctx_len"], tb["q_pos0"], hist)
    rc, word = dsa.get_error(clear=True)
    assert rc == 7 and word & 4, (rc, word)
    sc, got, want = _hist_pair(shape, tb)
    torch.testing.assert_close(got, want, rtol=0, atol=0)
    assert dsa.get_error()[0] == 0


def test_indexer_topk_handoff_against_oracle_decode32k():
    wl = workloads.get("decode32k")
    t = workloads.make_inputs(wl, DEV, seed=16, attention=False)
    shape = dsa.shape_from_workload(wl)
    _, got, _ = _hist_pair(shape, t)
    rows = _rows_all(wl.batch, 1)
    o_idx, o_sc = _oracle_idx_for(t, wl, rows)
    g_idx = got.reshape(-1, wl.topk).cpu().numpy()
    check_idx_valid(g_idx, _pos(H(t["q_pos0"]), rows), wl.topk)
    check_topk_near_ties(g_idx, o_idx, o_sc, wl.topk)


# --------------------------------------------------------------- attention --

def _oracle_idx_for(t, wl, rows):
    """Oracle indices (oracle scores -> oracle top-k) for the given rows."""
    sc = _oracle_scores(t, rows)
    pos = _pos(H(t["q_pos0"]), rows)
    return oracle.topk(np.where(np.isfinite(sc), sc, -np.inf).astype(np.float32), pos, wl.topk), sc


def _attn_oracle(t, idx, wl, rows, want_lse=False):
    v = H(t["v"]) if "v" in t else wl.d_v
    return oracle.sparse_attn(H(t["q"]), H(t["kv"]), idx, wl.sm_scale, v=v, rows=rows, want_lse=want_lse)


def _out_rows(out, rows, n_q):
    flat = out.reshape(-1, out.shape[2], out.shape[3]).float()
    sel = torch.tensor([b * n_q + t for b, t in rows], device=out.device, dtype=torch.long)
    return flat.index_select(0, sel).cpu().numpy().astype(np.float64)


def test_attention_tiny_fp32_on_oracle_indices():
    wl = workloads.get("tiny")
    t = workloads.make_inputs(wl, DEV, seed=0)
    rows = _rows_all(1, wl.n_q)
    idx, _ = _oracle_idx_for(t, wl, rows)
    shape = dsa.shape_from_workload(wl)
    idx_d = torch.from_numpy(idx).to(DEV).reshape(1, wl.n_q, wl.topk)
    lse = torch.empty(1, wl.n_q, wl.heads, dtype=torch.float32, device=DEV)
    out = dsa.sparse_mla_attn(shape, t["q"], t["kv"], idx_d, t["ctx_len"], v=t["v"], lse=lse)
    o, ol = _attn_oracle(t, idx, wl, rows, want_lse=True)
    np.testing.assert_allclose(_out_rows(out, rows, wl.n_q), o, rtol=0, atol=1e-5)
    np.testing.assert_allclose(lse.cpu().numpy().reshape(-1, wl.heads), ol, rtol=1e-5, atol=1e-5)


def test_attention_bf16_decode32k_on_oracle_indices():
    wl = workloads.get("decode32k")
    t = workloads.make_inputs(wl, DEV, seed=0)
    rows = _rows_all(wl.batch, 1)
    idx, _ = _oracle_idx_for(t, wl, rows)
    shape = dsa.shape_from_workload(wl)
    idx_d = torch.from_numpy(idx).to(DEV).reshape(wl.batch, 1, wl.topk)
    lse = torch.empty(wl.batch, 1, wl.heads, dtype=torch.float32, device=DEV)
    out = dsa.sparse_mla_attn(shape, t["q"], t["kv"], idx_d, t["ctx_len"], lse=lse)
    o, ol = _attn_oracle(t, idx, wl, rows, want_lse=True)
    err = np.abs(_out_rows(out, rows, 1) - o).max()
    assert err <= ATTN_ATOL_BF16, err
    np.testing.assert_allclose(lse.cpu().numpy().reshape(-1, wl.heads), ol, rtol=1e-4, atol=1e-4)


def test_attention_bf16_ragged_selection_and_padding():
    """Short rows (fewer than k selected, -1 padding), one key, unsorted
    indices, a length not a multiple of the gather tile."""
    wl = _custom("decode32k", batch=4, s_max=3000, ctx_len=(3000, 1, 77, 2900))
    t = workloads.make_inputs(wl, DEV, seed=4)
    g = np.random.default_rng(4)
    idx = np.full((4, wl.topk), -1, dtype=np.int32)
    for b, L in enumerate(wl.lengths()):
        n = min(wl.topk, L) if b != 3 else 1531
        idx[b, :n] = g.permutation(L)[:n]
    rows = _rows_all(4, 1)
    out = dsa.sparse_mla_attn(dsa.shape_from_workload(wl), t["q"], t["kv"],
                              torch.from_numpy(idx).to(DEV).reshape(4, 1, -1), t["ctx_len"])
    o = _attn_oracle(t, idx, wl, rows)
    err = np.abs(_out_rows(out, rows, 1) - o).max()
    assert err <= ATTN_ATOL_BF16, err


def test_attention_bf16_two_splits_per_query():
    """32 decode queries (the benchmark's batch): the split plan gives each
    query two splits, merged by the combine kernel.  Rows with an empty
    second split (at most 1024 selected keys) and a partial one, -1 padding,
    unsorted indices; output and lse against the oracle."""
    lengths = tuple([4096] * 28 + [100, 1024, 1500, 2049])
    wl = _custom("decode32k", batch=32, s_max=4096, ctx_len=lengths)
    t = workloads.make_inputs(wl, DEV, seed=18)
    g = np.random.default_rng(18)
    idx = np.full((32, wl.topk), -1, dtype=np.int32)
    for b, L in enumerate(lengths):
        n = min(wl.topk, L)
        idx[b, :n] = g.permutation(L)[:n]
    shape = dsa.shape_from_workload(wl)
    lse = torch.empty(32, 1, wl.heads, dtype=torch.float32, device=DEV)
    out = dsa.sparse_mla_attn(shape, t["q"], t["kv"], torch.from_numpy(idx).to(DEV).reshape(32, 1, -1),
                              t["ctx_len"], lse=lse)
    rows = _rows_all(32, 1)
    o, ol = _attn_oracle(t, idx, wl, rows, want_lse=True)
    err = np.abs(_out_rows(out, rows, 1) - o).max()
    assert err <= ATTN_ATOL_BF16, err
    np.testing.assert_allclose(lse.cpu().numpy().reshape(-1, wl.heads), ol, rtol=1e-4, atol=1e-4)
    assert dsa.get_error()[0] == 0


def test_attention_out_of_range_index_is_skipped_and_flagged():
    wl = _custom("decode32k", batch=2, s_max=1024, ctx_len=(1024, 512))
    t = workloads.make_inputs(wl, DEV, seed=6)
    idx = np.full((2, wl.topk), -1, dtype=np.int32)
    idx[0, :300] = np.arange(300)
    idx[1, :300] = np.arange(300)
    idx[1, 300] = 700                      # >= ctx_len[1] (but < s_max): skipped
    dsa.get_error(clear=True)
    out = dsa.sparse_mla_attn(dsa.shape_from_workload(wl), t["q"], t["kv"],
                              torch.from_numpy(idx).to(DEV).reshape(2, 1, -1), t["ctx_len"])
    rc, word = dsa.get_error(clear=True)
    assert rc == 6 and (word & 2), (rc, word)
    ok = idx.copy()
    ok[1, 300] = -1
    o = _attn_oracle(t, ok, wl, _rows_all(2, 1))
    assert np.abs(_out_rows(out, _rows_all(2, 1), 1) - o).max() <= ATTN_ATOL_BF16


# ----------------------------------------------------------------- forward --

def _forward_check(wl, t, rows, q_chunk=0, atol=ATTN_ATOL_BF16):
    shape = dsa.shape_from_workload(wl, q_chunk=q_chunk)
    idx_out = torch.empty(wl.batch, wl.n_q, wl.topk, dtype=torch.int32, device=DEV)
    out = dsa.forward(shape, t["q_idx"], t["k_idx"], t["w"], t["q"], t["kv"], t["ctx_len"], t["q_pos0"],
                      v=t.get("v"), idx_out=idx_out)
    o_idx, o_sc = _oracle_idx_for(t, wl, rows)
    g_idx = idx_out.reshape(-1, wl.topk).cpu().numpy()[[b * wl.n_q + tt for b, tt in rows]]
    check_idx_valid(g_idx, _pos(H(t["q_pos0"]), rows), wl.topk)
    check_topk_near_ties(g_idx, o_idx, o_sc, wl.topk)
    o = _attn_oracle(t, o_idx, wl, rows)
    err = np.abs(_out_rows(out, rows, wl.n_q) - o).max()
    assert err <= atol, err
    return out


def test_forward_tiny_fp32():
    wl = workloads.get("tiny")
    t = workloads.make_inputs(wl, DEV, seed=0)
    _forward_check(wl, t, _rows_all(1, wl.n_q), atol=1e-5)


def test_forward_tiny_fp32_chunked_rounds():
    wl = workloads.get("tiny")
    t = workloads.make_inputs(wl, DEV, seed=2)
    _forward_check(wl, t, _rows_all(1, wl.n_q), q_chunk=96, atol=1e-5)


def test_forward_bf16_decode32k():
    wl = workloads.get("decode32k")
    t = workloads.make_inputs(wl, DEV, seed=0)
    _forward_check(wl, t, _rows_all(wl.batch, 1))


def test_forward_bf16_prefill_chunked_two_sequences():
    wl = _custom("prefill8k", batch=2, n_q=640, s_max=2600, topk=256, ctx_len=(2600, 1900))
    t = workloads.make_inputs(wl, DEV, seed=8)
    t["q_pos0"] = torch.tensor([1960, 1260], dtype=torch.int32, device=DEV)
    rows = [(b, r) for b in range(2) for r in (0, 1, 100, 255, 256, 400, 639)]
    _forward_check(wl, t, rows, q_chunk=200)


def test_forward_host_buffers_match_device_call():
    wl = _custom("decode32k", batch=4, s_max=8192)
    t = workloads.make_inputs(wl, DEV, seed=11)
    shape = dsa.shape_from_workload(wl)
    dev_out = dsa.forward(shape, t["q_idx"], t["k_idx"], t["w"], t["q"], t["kv"], t["ctx_len"], t["q_pos0"])
    pin = lambda x: x.cpu().pin_memory()
    h_out = torch.empty(dev_out.shape, dtype=dev_out.dtype).pin_memory()
    dsa.forward_host(shape, pin(t["q_idx"]), pin(t["w"]), pin(t["q"]), pin(t["ctx_len"]), pin(t["q_pos0"]),
                     t["k_idx"], t["kv"], h_out)
    torch.testing.assert_close(h_out, dev_out.cpu(), rtol=0, atol=0)
    rows = _rows_all(4, 1)
    o_idx, _ = _oracle_idx_for(t, wl, rows)
    o = _attn_oracle(t, o_idx, wl, rows)
    assert np.abs(h_out.float().numpy().reshape(4, wl.heads, wl.d_v) - o).max() <= ATTN_ATOL_BF16


def test_forward_host_async_calls_in_flight_share_one_workspace():
    """Three asynchronous host-buffer steps on different inputs, enqueued back
    to back on one workspace (each output copy runs under the next step), then
    a synchronous one: every output equals the device-buffer call's."""
    wl = _custom("decode32k", batch=4, s_max=8192)
    shape = dsa.shape_from_workload(wl)
    ins = [workloads.make_inputs(wl, DEV, seed=20 + i) for i in range(3)]
    want = [dsa.forward(shape, t["q_idx"], t["k_idx"], t["w"], t["q"], t["kv"], t["ctx_len"], t["q_pos0"]).cpu()
            for t in ins]
    pin = lambda x: x.cpu().pin_memory()
    hin = [{k: pin(t[k]) for k in ("q_idx", "w", "q", "ctx_len", "q_pos0")} for t in ins]
    ws = torch.empty(dsa.workspace_bytes(shape, dsa.WS_FORWARD_HOST), dtype=torch.uint8, device=DEV)
    h_out = [torch.empty(want[0].shape, dtype=want[0].dtype).pin_memory() for _ in range(4)]
    done = [torch.cuda.Event() for _ in range(3)]
    torch.cuda.synchronize()
    for i, (t, h) in enumerate(zip(ins, hin)):
        dsa.forward_host_async(shape, h["q_idx"], h["w"], h["q"], h["ctx_len"], h["q_pos0"], t["k_idx"], t["kv"],
                               h_out[i], done=done[i], workspace=ws)
    h = hin[0]
    dsa.forward_host(shape, h["q_idx"], h["w"], h["q"], h["ctx_len"], h["q_pos0"], ins[0]["k_idx"], ins[0]["kv"],
                     h_out[3], workspace=ws)
    for i in range(3):
        done[i].synchronize()
        torch.testing.assert_close(h_out[i], want[i], rtol=0, atol=0)
    torch.testing.assert_close(h_out[3], want[0], rtol=0, atol=0)
    assert dsa.get_error()[0] == 0


# --------------------------------------------------------------------- FP8 --

def _codes_ok(g_code, o_code, quot):
    """Codes agree; where they differ, the oracle's unrounded value lies within
    1e-5 relative of the midpoint between the two neighbouring codes."""
    diff = g_code != o_code
    if not diff.any():
        return 0
    gv = oracle.e4m3_decode(g_code[diff])
    ov = oracle.e4m3_decode(o_code[diff])
    mid = 0.5 * (gv + ov)
    q = quot[diff]
    assert np.all(np.abs(q - mid) <= 1e-5 * np.maximum(np.abs(mid), 2.0 ** -9)), "e4m3 code mismatch"
    return int(diff.sum())


def test_hadamard_quant_matches_oracle():
    g = torch.Generator(device=DEV).manual_seed(3)
    x = (torch.randn(4096, 128, generator=g, device=DEV) / math.sqrt(128)).to(torch.bfloat16)
    x[7] = 0
    x8, sc = dsa.hadamard_quant_fp8(x)
    o_code, o_sc, quot = oracle.hadamard_quant(H(x))
    np.testing.assert_allclose(sc.cpu().numpy(), o_sc, rtol=2e-6, atol=0)
    assert sc[7].item() == 1.0
    n = _codes_ok(x8.cpu().numpy(), o_code, quot)
    assert n <= 64, n


def test_indexer_fp8_on_oracle_codes():
    """The FP8 indexer on the oracle's codes and scales equals the oracle's
    FP8 score (the dot product of e4m3 codes is exact in fp32)."""
    wl = _custom("decode32k", batch=3, s_max=4000, ctx_len=(4000, 2500, 129))
    t = workloads.make_inputs(wl, "cpu", seed=5, attention=False)
    qc, qs, _ = oracle.hadamard_quant(H(t["q_idx"]))
    kc, ks, _ = oracle.hadamard_quant(H(t["k_idx"]))
    shape = dsa.shape_from_workload(wl).replace(idx_dtype=dsa.DSA_E4M3)
    d = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(DEV)
    sc = dsa.indexer_scores(shape, d(qc), d(kc), d(H(t["w"])), d(H(t["ctx_len"])), d(H(t["q_pos0"])),
                            q_scale=d(qs), k_scale=d(ks))
    rows = _rows_all(3, 1)
    ora = oracle.indexer_scores_fp8(qc, qs, kc, ks, H(t["w"]), H(t["ctx_len"]), H(t["q_pos0"]), rows=rows)
    check_scores(_scores_for_rows(sc, rows), ora, list(wl.lengths()))


def _recall(a, b, k):
    return [len(set(a[r][a[r] >= 0]) & set(b[r][b[r] >= 0])) / k for r in range(a.shape[0])]


def test_forward_fp8_without_rescoring_matches_oracle_fp8_path():
    """FP8 indexer end to end, selecting on the FP8 scores alone
    (idx_rescore = 0).  The GPU's selection reproduces the oracle's own FP8
    path (rotate, per-row e4m3 codes, scores, top-k) -- sets equal except
    where a code sits on a rounding boundary.  Its recall against the bf16
    oracle is that of e4m3 with per-row scales on these gaussian inputs
    (about 0.965), below the 0.99 bar that the re-scored step below meets; it
    is asserted here as a regression bound.  The attention output equals the
    oracle's attention over the GPU's own selection."""
    wl = _custom("decode32k", batch=4, s_max=32768)
    t = workloads.make_inputs(wl, DEV, seed=12)
    k8, ks = dsa.hadamard_quant_fp8(t["k_idx"])
    shape = dsa.shape_from_workload(wl).replace(idx_dtype=dsa.DSA_E4M3, idx_rescore=0)
    idx_out = torch.empty(wl.batch, 1, wl.topk, dtype=torch.int32, device=DEV)
    out = dsa.forward(shape, t["q_idx"], k8, t["w"], t["q"], t["kv"], t["ctx_len"], t["q_pos0"], k_scale=ks,
                      idx_out=idx_out)
    rows = _rows_all(wl.batch, 1)
    o_idx, _ = _oracle_idx_for(t, wl, rows)
    h = {k: H(v) for k, v in t.items()}
    qc, qs, _ = oracle.hadamard_quant(h["q_idx"])
    kc, ks_o, _ = oracle.hadamard_quant(h["k_idx"])
    s8 = oracle.indexer_scores_fp8(qc, qs, kc, ks_o, h["w"], h["ctx_len"], h["q_pos0"], rows=rows)
    o8_idx = oracle.topk(s8.astype(np.float32), _pos(h["q_pos0"], rows), wl.topk)
    g_idx = idx_out.reshape(-1, wl.topk).cpu().numpy()
    assert min(_recall(g_idx, o8_idx, wl.topk)) >= 0.995
    g_rec, o_rec = _recall(g_idx, o_idx, wl.topk), _recall(o8_idx, o_idx, wl.topk)
    assert abs(np.mean(g_rec) - np.mean(o_rec)) <= 0.01, (g_rec, o_rec)
    assert min(g_rec) >= 0.95, g_rec
    o = _attn_oracle(t, g_idx, wl, rows)
    assert np.abs(_out_rows(out, rows, 1) - o).max() <= ATTN_ATOL_BF16


def test_indexer_rescore_on_listed_keys():
    """dsa_indexer_rescore on ascending candidate lists of several lengths
    (fewer candidates than listed for a short sequence, a list cut by the
    causal limit): the scores of the listed keys equal the oracle's bf16
    scores at those keys (1e-3 rule, rms over the full oracle row)."""
    wl = _custom("decode32k", batch=3, s_max=6000, ctx_len=(6000, 3000, 700))
    t = workloads.make_inputs(wl, DEV, seed=13, attention=False)
    n_cand, ld = 1000, 1004
    g = np.random.default_rng(13)
    cand = np.full((3, 1, ld), -1, dtype=np.int32)
    for b, L in enumerate(wl.lengths()):
        n = min(n_cand, L)
        cand[b, 0, :n] = np.sort(g.choice(L, size=n, replace=False))
    shape = dsa.shape_from_workload(wl)
    cand_d = torch.from_numpy(cand).to(DEV)
    sc = dsa.indexer_rescore(shape, t["q_idx"], t["k_idx"], t["w"], cand_d, n_cand, t["ctx_len"], t["q_pos0"])
    rows = _rows_all(3, 1)
    ora = _oracle_scores(t, rows)
    got = sc.reshape(3, -1).cpu().numpy()
    for r, L in enumerate(wl.lengths()):
        n = min(n_cand, L)
        sel = cand[r, 0, :n]
        g_r = got[r:r + 1, :n]
        o_r = ora[r:r + 1, sel]
        tol = 1e-3 * (np.abs(o_r) + rms_finite(ora[r]))
        assert np.all(np.abs(g_r - o_r) <= tol), r
    assert dsa.get_error()[0] == 0


def test_topk_candidates_exact_on_ties():
    """dsa_topk_candidates: top-k among listed keys, bit-exact against the
    oracle's top-k over the list (ties toward the earlier entry, which is the
    lower key index), mapped through the list; rows with fewer listed
    candidates than k, and a list longer than the causal limit."""
    g = np.random.default_rng(14)
    B, n_cand, ld, k = 5, 3072, 3072, 2048
    ctx = [131072, 131072, 2500, 131072, 1000]
    pos0 = [c - 1 for c in ctx]
    cand = np.full((B, 1, ld), -1, dtype=np.int32)
    for b in range(B):
        n = min(n_cand, ctx[b])
        cand[b, 0, :n] = np.sort(g.choice(ctx[b], size=n, replace=False))
    cs = (g.integers(-30, 30, size=(B, 1, ld)).astype(np.float32) * 0.125)
    cs[1, 0] = np.float32(0.5)                       # all equal
    shape = dsa.make_shape(B, 1, 131072, topk=k)
    got = dsa.topk_candidates(shape, torch.from_numpy(cs).to(DEV), torch.from_numpy(cand).to(DEV), n_cand,
                              torch.tensor(ctx, dtype=torch.int32, device=DEV),
                              torch.tensor(pos0, dtype=torch.int32, device=DEV)).cpu().numpy().reshape(B, k)
    for b in range(B):
        n = min(n_cand, pos0[b] + 1)
        slots = oracle.topk(cs[b:b + 1, 0, :n], np.array([n - 1], dtype=np.int32), k)[0]
        want = np.where(slots >= 0, cand[b, 0, np.maximum(slots, 0)], -1)
        np.testing.assert_array_equal(got[b], want)


def _fp8_rescored_case(wl, t, picked):
    """Run the e4m3 step with re-scoring on all of wl's sequences; check the
    picked ones against the bf16 oracle: recall >= 0.99 of the oracle's
    top-k, the selection equal to the oracle's top-k over the oracle's own
    FP8 candidates up to near-ties of the k-th bf16 score, and the output
    within 3e-2 of the oracle's attention over the bf16 oracle selection."""
    k8, ks = dsa.hadamard_quant_fp8(t["k_idx"])
    shape = dsa.shape_from_workload(wl).replace(idx_dtype=dsa.DSA_E4M3, idx_rescore=1024)
    idx_out = torch.empty(wl.batch, 1, wl.topk, dtype=torch.int32, device=DEV)
    out = dsa.forward(shape, t["q_idx"], k8, t["w"], t["q"], t["kv"], t["ctx_len"], t["q_pos0"], k_scale=ks,
                      idx_out=idx_out, k_rescore=t["k_idx"])
    torch.cuda.synchronize()
    assert dsa.get_error()[0] == 0
    sub = {k: t[k][picked].contiguous() for k in ("q_idx", "k_idx", "w", "q", "kv", "ctx_len", "q_pos0")}
    rows = [(i, 0) for i in range(len(picked))]
    o_idx, o_sc = _oracle_idx_for(sub, wl, rows)
    g_idx = idx_out.reshape(wl.batch, wl.topk)[picked].cpu().numpy()
    check_idx_valid(g_idx, _pos(H(sub["q_pos0"]), rows), wl.topk)
    rec = _recall(g_idx, o_idx, wl.topk)
    assert min(rec) >= 0.99, rec
    # the oracle's own re-scored selection: FP8 top-(k + 1024), then the bf16
    # top-k among them
    h = {k: H(v) for k, v in sub.items()}
    qc, qs, _ = oracle.hadamard_quant(h["q_idx"])
    kc8, ks_o, _ = oracle.hadamard_quant(h["k_idx"])
    s8 = oracle.indexer_scores_fp8(qc, qs, kc8, ks_o, h["w"], h["ctx_len"], h["q_pos0"], rows=rows)
    pos = _pos(h["q_pos0"], rows)
    cand = oracle.topk(s8.astype(np.float32), pos, wl.topk + 1024)
    want = np.full_like(o_idx, -1)
    for r in range(len(rows)):
        c = cand[r][cand[r] >= 0]
        cs = np.where(np.isfinite(o_sc[r, c]), o_sc[r, c], -np.inf).astype(np.float32)
        slots = oracle.topk(cs[None, :], np.array([c.size - 1], dtype=np.int32), wl.topk)[0]
        want[r] = np.where(slots >= 0, c[np.maximum(slots, 0)], -1)
    check_topk_near_ties(g_idx, want, o_sc, wl.topk)
    o = _attn_oracle(sub, o_idx, wl, rows)
    got = out[picked].float().cpu().numpy().reshape(len(picked), wl.heads, wl.d_v).astype(np.float64)
    err = np.abs(got - o).max()
    assert err <= 3e-2, err
    return rec, err


def test_forward_fp8_rescored_meets_bf16_bar():
    wl = _custom("decode32k", batch=4, s_max=32768)
    t = workloads.make_inputs(wl, DEV, seed=12)
    _fp8_rescored_case(wl, t, [0, 1, 2, 3])


@pytest.mark.slow
def test_forward_fp8_rescored_decode128k_full_size():
    """The e4m3 benchmark configuration (32 queries at 131072 keys, k = 2048,
    1024 re-scored extra candidates): the oracle checks three sequences."""
    wl = workloads.get("decode128k_fp8")
    t = workloads.make_inputs(wl, DEV, seed=0)
    _fp8_rescored_case(wl, t, [0, 16, 31])


@pytest.mark.parametrize("case", ["decode_split", "prefill_rounds", "fp8_rescored"])
def test_forward_poisoned_buffers_change_nothing(case):
    """Race-detection stand-in: the step run on a workspace, output and lse
    pre-filled with 0xFF bytes (NaN in every float view) must equal, bit for
    bit, the step run on zeroed buffers, with every output element written:
    a kernel that reads scratch nobody wrote this call, or leaves part of an
    output unwritten (e.g. a split the combine skips), fails here."""
    if case == "decode_split":
        wl = _custom("decode32k", batch=3, s_max=9000, ctx_len=(9000, 2100, 5000))
        extra, q_chunk = {}, 0
    elif case == "prefill_rounds":
        wl = _custom("prefill8k", batch=1, n_q=700, s_max=2500, topk=512, ctx_len=(2500,))
        extra, q_chunk = {}, 256
    else:
        wl = _custom("decode32k", batch=2, s_max=6000)
        extra, q_chunk = {"idx_dtype": dsa.DSA_E4M3, "idx_rescore": 1024}, 0
    t = workloads.make_inputs(wl, DEV, seed=17)
    if case == "prefill_rounds":
        t["q_pos0"] = torch.tensor([2500 - 700], dtype=torch.int32, device=DEV)
    shape = dsa.shape_from_workload(wl, q_chunk=q_chunk).replace(**extra)
    k_idx, k_scale, k_ref = t["k_idx"], None, None
    if case == "fp8_rescored":
        k_idx, k_scale = dsa.hadamard_quant_fp8(t["k_idx"])
        k_ref = t["k_idx"]
    nbytes = dsa.workspace_bytes(shape, dsa.WS_FORWARD)
    res = []
    for fill in (0x00, 0xFF):
        ws = torch.full((nbytes,), fill, dtype=torch.uint8, device=DEV)
        out = torch.empty(wl.batch, wl.n_q, wl.heads, wl.d_v, dtype=torch.bfloat16, device=DEV)
        out.view(torch.int16).fill_(-1 if fill else 0)
        lse = torch.empty(wl.batch, wl.n_q, wl.heads, dtype=torch.float32, device=DEV)
        lse.view(torch.int32).fill_(-1 if fill else 0)
        idx = torch.full((wl.batch, wl.n_q, wl.topk), -7 if fill else 7, dtype=torch.int32, device=DEV)
        dsa.forward(shape, t["q_idx"], k_idx, t["w"], t["q"], t["kv"], t["ctx_len"], t["q_pos0"], out=out, lse=lse,
                    idx_out=idx, workspace=ws, k_scale=k_scale, k_rescore=k_ref)
        torch.cuda.synchronize()
        res.append((out.clone(), lse.clone(), idx.clone()))
    for a, b in zip(res[0], res[1]):
        assert torch.equal(a.view(torch.uint8) if a.dtype == torch.bfloat16 else a,
                           b.view(torch.uint8) if b.dtype == torch.bfloat16 else b)
    assert torch.isfinite(res[1][0].float()).all() and torch.isfinite(res[1][1]).all()
    assert dsa.get_error()[0] == 0


@pytest.mark.slow
def test_forward_decode128k_full_size_sampled_sequences():
    """The benchmark's configuration (32 queries at 131072 keys, k = 2048, same
    split plan): the step runs on all 32 sequences; the oracle checks three."""
    wl = workloads.get("decode128k")
    t = workloads.make_inputs(wl, DEV, seed=0)
    shape = dsa.shape_from_workload(wl)
    idx_out = torch.empty(wl.batch, 1, wl.topk, dtype=torch.int32, device=DEV)
    out = dsa.forward(shape, t["q_idx"], t["k_idx"], t["w"], t["q"], t["kv"], t["ctx_len"], t["q_pos0"],
                      idx_out=idx_out)
    torch.cuda.synchronize()
    picked = [0, 13, 31]
    sub = {k: t[k][picked].contiguous() for k in ("q_idx", "k_idx", "w", "q", "kv", "ctx_len", "q_pos0")}
    rows = [(i, 0) for i in range(len(picked))]
    o_idx, o_sc = _oracle_idx_for(sub, wl, rows)
    g_idx = idx_out.reshape(wl.batch, wl.topk)[picked].cpu().numpy()
    check_idx_valid(g_idx, _pos(H(sub["q_pos0"]), rows), wl.topk)
    check_topk_near_ties(g_idx, o_idx, o_sc, wl.topk)
    o = _attn_oracle(sub, o_idx, wl, rows)
    got = out[picked].float().cpu().numpy().reshape(len(picked), wl.heads, wl.d_v).astype(np.float64)
    assert np.abs(got - o).max() <= ATTN_ATOL_BF16
