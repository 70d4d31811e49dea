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


def test_topk_gaussian_decode128k_shape():
    g = np.random.default_rng(9)
    B, S, k = 32, 131072, 2048
    sc = g.standard_normal((B, 1, S)).astype(np.float32)
    _topk_case(B, 1, S, k, [S] * B, [S - 1] * B, sc)


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


def test_forward_fp8_matches_oracle_fp8_path():
    """FP8 indexer end to end.  The GPU's selection reproduces the oracle's own
    FP8 path (rotate, per-row e4m3 codes, scores, top-k) -- sets equal except
    where a code sits on a rounding boundary -- so its recall against the bf16
    oracle equals the oracle FP8 path's recall.  That recall is a property of
    E4M3 with per-row scales on these gaussian inputs (about 0.965 here), below
    the 0.99 aimed for; the attention output stays within 3e-2 of the bf16
    oracle's."""
    wl = _custom("decode32k", batch=4, s_max=32768)
    t = workloads.make_inputs(wl, DEV, seed=12)
    k8, ks = dsa.hadamard_quant_fp8(t["k_idx"])
    shape = dsa.shape_from_workload(wl).replace(idx_dtype=dsa.DSA_E4M3)
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
    rec = lambda a, b, r: len(set(a[r]) & set(b[r])) / wl.topk
    same = [rec(g_idx, o8_idx, r) for r in range(wl.batch)]
    assert min(same) >= 0.995, same
    g_rec = [rec(g_idx, o_idx, r) for r in range(wl.batch)]
    o_rec = [rec(o8_idx, o_idx, r) for r in range(wl.batch)]
    assert abs(np.mean(g_rec) - np.mean(o_rec)) <= 0.01, (g_rec, o_rec)
    assert torch.isfinite(out.float()).all()


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
