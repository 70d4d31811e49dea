"""Pins of the CPU oracle to things other than itself (no GPU needed).

Each test ties one oracle function to a library routine, a closed form, an
invariant, a special case, or a brute force, chosen so that a dropped term,
a wrong sign or index, or a transposed operand fails at least one of them.
Sources: DeepSeek-V3.2 model doc (Transformers), section "DeepSeek Sparse
Attention (DSA)" items 1-2 and section DeepseekV32Config; OCP OFP8 spec for
E4M3.
"""
import json
import math
import os

import numpy as np
import pytest
import scipy.linalg
import torch
import torch.nn.functional as F

import oracle
import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _bf16_bits(x: torch.Tensor):
    return x.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


# ------------------------------------------------------------------ indexer --

def _idx_case(B=2, n_q=5, S=40, H=3, D=16, seed=0, ctx=None, pos0=None):
    g = np.random.default_rng(seed)
    q = g.standard_normal((B, n_q, H, D)).astype(np.float32)
    k = g.standard_normal((B, S, D)).astype(np.float32)
    w = g.standard_normal((B, n_q, H)).astype(np.float32)
    ctx = np.array(ctx if ctx is not None else [S] * B, dtype=np.int32)
    pos0 = np.array(pos0 if pos0 is not None else [c - n_q for c in ctx], dtype=np.int32)
    return q, k, w, ctx, pos0


def test_indexer_single_head_is_relu_of_matmul():
    """H = 1, w = 1: scores reduce to ReLU(Q K^T) (BLAS matmul), causal, ragged."""
    q, k, w, ctx, pos0 = _idx_case(H=1, ctx=[40, 23], pos0=[10, 18])
    w[:] = 1.0
    out = oracle.indexer_scores(q, k, w, ctx, pos0)
    r = 0
    for b in range(2):
        dense = np.maximum(q[b, :, 0, :].astype(np.float64) @ k[b].astype(np.float64).T, 0.0)
        for t in range(q.shape[1]):
            p = pos0[b] + t
            L = ctx[b]
            np.testing.assert_allclose(out[r, :p + 1], dense[t, :p + 1], rtol=1e-12, atol=1e-12)
            assert np.all(np.isneginf(out[r, p + 1:L]))
            assert np.all(np.isnan(out[r, L:]))
            r += 1


def test_indexer_one_hot_weight_selects_head():
    q, k, w, ctx, pos0 = _idx_case(H=4)
    for j in range(4):
        wj = np.zeros_like(w)
        wj[..., j] = 1.0
        out = oracle.indexer_scores(q, k, wj, ctx, pos0)
        r = 0
        for b in range(q.shape[0]):
            dense = np.maximum(q[b, :, j, :].astype(np.float64) @ k[b].astype(np.float64).T, 0.0)
            for t in range(q.shape[1]):
                p = pos0[b] + t
                np.testing.assert_allclose(out[r, :p + 1], dense[t, :p + 1], rtol=1e-12, atol=1e-12)
                r += 1


def test_indexer_linear_and_odd_in_weights():
    """The weights multiply outside the ReLU: I(w1 + w2) = I(w1) + I(w2), I(-w) = -I(w), I(0) = 0."""
    q, k, w, ctx, pos0 = _idx_case(H=5, seed=3)
    w2 = np.random.default_rng(9).standard_normal(w.shape).astype(np.float32)
    a = oracle.indexer_scores(q, k, w, ctx, pos0)
    b = oracle.indexer_scores(q, k, w2, ctx, pos0)
    ab = oracle.indexer_scores(q, k, (w.astype(np.float64) + w2).astype(np.float32), ctx, pos0)
    fin = np.isfinite(a)
    # w + w2 rounded to fp32: allow that rounding
    np.testing.assert_allclose(ab[fin], a[fin] + b[fin], rtol=1e-6, atol=1e-6)
    neg = oracle.indexer_scores(q, k, -w, ctx, pos0)
    np.testing.assert_array_equal(neg[fin], -a[fin])
    zero = oracle.indexer_scores(q, k, np.zeros_like(w), ctx, pos0)
    assert np.all(zero[fin] == 0.0)


def test_indexer_relu_is_per_head_not_on_sum():
    """ReLU applies to each head's dot product: with w = 1 on two heads whose dots
    are +a and -b, the score is a, not max(0, a - b)."""
    D = 4
    q = np.zeros((1, 1, 2, D), np.float32)
    q[0, 0, 0, 0] = 2.0
    q[0, 0, 1, 1] = 3.0
    k = np.zeros((1, 1, D), np.float32)
    k[0, 0, 0] = 1.0
    k[0, 0, 1] = -1.0
    w = np.ones((1, 1, 2), np.float32)
    out = oracle.indexer_scores(q, k, w, [1], [0])
    assert out[0, 0] == 2.0


def test_indexer_scale_homogeneous_and_bf16_widening_exact():
    q, k, w, ctx, pos0 = _idx_case(seed=5)
    a = oracle.indexer_scores(q, k, w, ctx, pos0, scale=1.0)
    b = oracle.indexer_scores(q, k, w, ctx, pos0, scale=0.25)
    fin = np.isfinite(a)
    np.testing.assert_allclose(b[fin], 0.25 * a[fin], rtol=1e-13, atol=1e-14)
    qt, kt = torch.from_numpy(q), torch.from_numpy(k)
    qb, kb = qt.to(torch.bfloat16), kt.to(torch.bfloat16)
    via_bits = oracle.indexer_scores(_bf16_bits(qt), _bf16_bits(kt), w, ctx, pos0)
    via_f32 = oracle.indexer_scores(qb.float().numpy(), kb.float().numpy(), w, ctx, pos0)
    np.testing.assert_array_equal(via_bits[fin], via_f32[fin])


def test_indexer_diagonal_included():
    """'Previous keys' is read as s <= p: the query's own key is scored."""
    q, k, w, ctx, pos0 = _idx_case(B=1, n_q=1, S=8, H=1, D=4, ctx=[8], pos0=[7])
    w[:] = 1.0
    k[0, 7] = q[0, 0, 0]          # own key: dot = |q|^2 > 0
    out = oracle.indexer_scores(q, k, w, ctx, pos0)
    assert out[0, 7] == pytest.approx(float(np.dot(q[0, 0, 0].astype(np.float64), q[0, 0, 0])), rel=1e-12)


# ----------------------------------------------------------------- hadamard --

@pytest.mark.parametrize("n", [2, 8, 32, 128])
def test_hadamard_matches_scipy(n):
    x = np.random.default_rng(n).standard_normal((7, n))
    H = scipy.linalg.hadamard(n).astype(np.float64) / math.sqrt(n)
    np.testing.assert_allclose(oracle.hadamard(x), x @ H.T, rtol=0, atol=1e-13)


def test_hadamard_orthogonal_and_involution():
    n = 128
    H = oracle.hadamard(np.eye(n))          # rows: H e_i
    Hs = scipy.linalg.hadamard(n).astype(np.float64)
    np.testing.assert_array_equal(Hs @ Hs.T, n * np.eye(n))      # +-1 matrix, exact
    np.testing.assert_allclose(H @ H.T, np.eye(n), atol=1e-14)
    g = np.random.default_rng(1)
    q, k = g.standard_normal((50, n)), g.standard_normal((50, n))
    Hq, Hk = oracle.hadamard(q), oracle.hadamard(k)
    # Hq . Hk = q . k (DSA item 1)
    np.testing.assert_allclose((Hq * Hk).sum(1), (q * k).sum(1), rtol=0, atol=1e-12)
    np.testing.assert_allclose(oracle.hadamard(Hq), q, atol=1e-13)
    e0 = np.zeros(n)
    e0[0] = 1
    np.testing.assert_allclose(oracle.hadamard(e0[None])[0], np.full(n, 1 / math.sqrt(n)), atol=1e-15)


# --------------------------------------------------------------------- e4m3 --

def test_e4m3_spec_points():
    rows = [l.split() for l in open(os.path.join(GOLDEN, "e4m3_spec_points.txt")) if l.strip() and not l.startswith("#")]
    for code_s, val_s in rows:
        code, val = int(code_s, 16), float(val_s)
        dec = oracle.e4m3_decode(np.array([code], np.uint8))[0]
        assert dec == val and math.copysign(1, dec) == math.copysign(1, val), (code_s, dec, val)
        assert oracle.e4m3_encode(np.array([val]))[0] == code


def test_e4m3_decode_matches_torch_all_codes():
    codes = np.arange(256, dtype=np.uint8)
    ours = oracle.e4m3_decode(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan) and nan.sum() == 2
    np.testing.assert_array_equal(ours[~nan], ref[~nan])


def test_e4m3_encode_matches_torch_rne_on_all_bf16():
    """Every finite bf16 value: round-to-nearest-even agrees with torch's cast
    within range; beyond +-448 the oracle saturates (satfinite)."""
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    x = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64)
    x = x[torch.isfinite(x)]
    ours = oracle.e4m3_encode(x.numpy())
    inr = x.abs() <= 448
    ref = x[inr].to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(ours[inr.numpy()], ref)
    big = (~inr).numpy()
    assert np.all((ours[big] & 0x7F) == 0x7E)
    assert np.all((ours[big] >> 7) == (x.numpy()[big] < 0))


def test_e4m3_ties_to_even():
    # 1 + 1/16 is halfway between 1.0 (m=0) and 1.125 (m=1): even -> 1.0
    # 1 + 3/16 is halfway between 1.125 (m=1) and 1.25 (m=2): even -> 1.25
    # 2^-10 is halfway between 0 and the smallest subnormal 2^-9: even -> 0
    vals = np.array([1.0625, 1.1875, 2.0 ** -10, 3 * 2.0 ** -10, 464.0, -500.0])
    dec = oracle.e4m3_decode(oracle.e4m3_encode(vals))
    np.testing.assert_array_equal(dec, [1.0, 1.25, 0.0, 2.0 ** -8, 448.0, -448.0])


def test_hadamard_quant_exact_on_representable_rows():
    """x = H y with y on the e4m3 grid and max|y| = 448: sigma = 1, codes = y."""
    g = np.random.default_rng(2)
    n = 128
    codes = g.integers(0, 256, size=(20, n)).astype(np.uint8)
    codes[(codes & 0x7F) == 0x7F] = 0x3C         # drop NaN codes
    codes[:, 5] = 0x7E                            # amax 448
    y = oracle.e4m3_decode(codes)
    x = oracle.hadamard(y).astype(np.float32)     # fp32 storage rounds x slightly
    c2, sigma, quot = oracle.hadamard_quant(x)
    assert np.all(np.abs(sigma - 1.0) < 1e-6)
    dec = oracle.e4m3_decode(c2)
    np.testing.assert_array_equal(dec, y)


def test_fp8_indexer_exact_on_representable_inputs():
    """With codes and scales given directly, the FP8 score equals the plain
    score of the decoded values times the scales."""
    g = np.random.default_rng(4)
    B, n_q, H, D, S = 1, 3, 4, 128, 20
    qc = g.integers(0, 0x7E, size=(B, n_q, H, D)).astype(np.uint8)
    kc = g.integers(0, 0x7E, size=(B, S, D)).astype(np.uint8)
    qs = np.full((B, n_q, H), 0.5, np.float32)
    ks = np.full((B, S), 0.25, np.float32)
    w = g.standard_normal((B, n_q, H)).astype(np.float32)
    ctx, pos0 = [S], [S - n_q]
    a = oracle.indexer_scores_fp8(qc, qs, kc, ks, w, ctx, pos0)
    qd = oracle.e4m3_decode(qc) * 0.5
    kd = oracle.e4m3_decode(kc) * 0.25
    b = oracle.indexer_scores(qd.astype(np.float32), kd.astype(np.float32), w, ctx, pos0)
    fin = np.isfinite(b)
    np.testing.assert_allclose(a[fin], b[fin], rtol=1e-12, atol=1e-12)
    np.testing.assert_array_equal(np.isneginf(a), np.isneginf(b))


def test_fp8_indexer_within_quantisation_bound():
    """Rotation + per-row e4m3 coding perturbs each rotated element by at most
    2^-4 relative (half a 3-bit-mantissa ulp) or 2^-10 sigma absolute
    (subnormals); the head-summed score stays within the propagated bound."""
    g = np.random.default_rng(6)
    B, n_q, H, D, S = 1, 2, 8, 128, 64
    q = (g.standard_normal((B, n_q, H, D)) / math.sqrt(D)).astype(np.float32)
    k = (g.standard_normal((B, S, D)) / math.sqrt(D)).astype(np.float32)
    w = g.standard_normal((B, n_q, H)).astype(np.float32)
    ctx, pos0 = [S], [S - n_q]
    exact = oracle.indexer_scores(q, k, w, ctx, pos0)
    qc, qs, _ = oracle.hadamard_quant(q)
    kc, ks, _ = oracle.hadamard_quant(k)
    approx = oracle.indexer_scores_fp8(qc, qs, kc, ks, w, ctx, pos0)
    Hq, Hk = oracle.hadamard(q.astype(np.float64)), oracle.hadamard(k.astype(np.float64))
    dq = np.abs(Hq) * 2.0 ** -4 + qs[..., None] * 2.0 ** -10
    dk = np.abs(Hk) * 2.0 ** -4 + ks[..., None] * 2.0 ** -10
    for t in range(n_q):
        p = pos0[0] + t
        for s in range(p + 1):
            bound = 0.0
            for h in range(H):
                e = (np.abs(Hq[0, t, h]) * dk[0, s] + np.abs(Hk[0, s]) * dq[0, t, h] + dq[0, t, h] * dk[0, s]).sum()
                bound += abs(w[0, t, h]) * e
            assert abs(approx[t, s] - exact[t, s]) <= bound * (1 + 1e-9) + 1e-12


# -------------------------------------------------------------------- top-k --

def _brute_topk(row, p, k):
    cand = np.arange(p + 1)
    order = np.lexsort((cand, -row[: p + 1].astype(np.float64)))   # score desc, index asc
    keep = np.sort(cand[order[: min(k, p + 1)]])
    return np.concatenate([keep, -np.ones(k - keep.size, np.int64)])


@pytest.mark.parametrize("seed", range(6))
def test_topk_matches_lexsort_bruteforce(seed):
    g = np.random.default_rng(seed)
    nrows, S, k = 12, 64, 9
    # few distinct values -> many exact ties
    scores = g.integers(-4, 5, size=(nrows, S)).astype(np.float32) * 0.5
    scores[0] = 0.0                      # all equal
    scores[1, ::2] = -0.0                # signed zeros compare equal
    pos = g.integers(0, S, size=nrows).astype(np.int32)
    pos[2] = 3                           # fewer candidates than k
    idx = oracle.topk(scores, pos, k)
    for r in range(nrows):
        np.testing.assert_array_equal(idx[r], _brute_topk(scores[r], pos[r], k))


def test_topk_matches_bruteforce_on_arbitrary_finite_floats():
    """Property test: any finite fp32 values (subnormals, signed zeros, the
    extremes, heavy repetition), any row length, k and causal position."""
    hyp = pytest.importorskip("hypothesis")
    st = hyp.strategies

    finite = st.floats(width=32, allow_nan=False, allow_infinity=False)
    pool = st.lists(finite, min_size=1, max_size=6)  # few distinct values -> ties

    @hyp.settings(max_examples=300, deadline=None, derandomize=True)
    @hyp.given(data=st.data())
    def check(data):
        S = data.draw(st.integers(1, 48))
        vals = data.draw(pool)
        row = np.array(data.draw(st.lists(st.sampled_from(vals), min_size=S, max_size=S)), np.float32)
        p = data.draw(st.integers(0, S - 1))
        k = data.draw(st.integers(1, S + 3))
        got = oracle.topk(row[None, :], np.array([p], np.int32), k)[0]
        np.testing.assert_array_equal(got, _brute_topk(row, p, k))

    check()


def test_topk_invariants():
    g = np.random.default_rng(11)
    S, k = 50, 16
    scores = g.standard_normal((S, S)).astype(np.float32)
    pos = np.arange(S, dtype=np.int32)
    idx = oracle.topk(scores, pos, k)
    for r in range(S):
        sel = idx[r][idx[r] >= 0]
        assert sel.size == min(k, r + 1)
        assert sel.max() <= r and np.all(np.diff(sel) > 0)
        if r + 1 <= k:
            np.testing.assert_array_equal(sel, np.arange(r + 1))
        else:
            thr = np.sort(scores[r, : r + 1])[::-1][k - 1]
            assert np.all(scores[r, sel] >= thr)
    all_eq = np.zeros((1, S), np.float32)
    np.testing.assert_array_equal(oracle.topk(all_eq, [S - 1], k)[0], np.arange(k))


def test_topk_rejects_nonfinite():
    s = np.zeros((1, 8), np.float32)
    s[0, 3] = np.nan
    with pytest.raises(ValueError):
        oracle.topk(s, [7], 4)


# ---------------------------------------------------------------- attention --

def _mha_case(B=1, L=24, H=2, KVH=2, d=16, dv=16, seed=0):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, L, H, d, generator=g)
    k = torch.randn(B, L, KVH, d, generator=g)
    v = torch.randn(B, L, KVH, dv, generator=g)
    return q, k, v


def test_attention_full_selection_equals_causal_sdpa_mha():
    """index_topk >= L: sparse attention is dense causal attention (DSA item 2)."""
    L, scale = 24, 1 / math.sqrt(16)
    q, k, v = _mha_case(L=L)
    idx = np.tile(np.arange(L, dtype=np.int32), (L, 1))
    idx = np.where(idx <= np.arange(L)[:, None], idx, -1).astype(np.int32)
    out, lse = oracle.sparse_attn(q.numpy(), k.numpy(), idx, scale, v=v.numpy(), want_lse=True)
    ref = F.scaled_dot_product_attention(q.double().transpose(1, 2), k.double().transpose(1, 2),
                                         v.double().transpose(1, 2), is_causal=True, scale=scale)
    ref = ref.transpose(1, 2)[0].numpy()      # [L, H, dv]
    np.testing.assert_allclose(out, ref, rtol=1e-11, atol=1e-12)
    logits = torch.einsum("thd,shd->ths", q.double()[0], k.double()[0]) * scale
    mask = torch.arange(L)[None, None, :] > torch.arange(L)[:, None, None]
    ref_lse = torch.logsumexp(logits.masked_fill(mask, -math.inf), dim=-1).numpy()
    np.testing.assert_allclose(lse, ref_lse, rtol=1e-12, atol=1e-12)


def test_attention_full_selection_equals_sdpa_absorbed_mla():
    """Absorbed MLA form: one shared latent row (d_qk) per token, value = its
    first d_v columns, every head reads the same row."""
    g = torch.Generator().manual_seed(3)
    B, L, H, dqk, dv = 2, 20, 4, 48, 32
    scale = 1 / math.sqrt(24)
    q = torch.randn(B, L, H, dqk, generator=g)
    kv = torch.randn(B, L, dqk, generator=g)
    idx = np.tile(np.arange(L, dtype=np.int32), (B * L, 1))
    pos = np.tile(np.arange(L), B)
    idx = np.where(idx <= pos[:, None], idx, -1).astype(np.int32)
    out = oracle.sparse_attn(q.numpy(), kv.numpy(), idx, scale, v=dv)
    kk = kv.double()[:, None].expand(B, H, L, dqk)
    vv = kv.double()[:, None, :, :dv].expand(B, H, L, dv)
    ref = F.scaled_dot_product_attention(q.double().transpose(1, 2), kk, vv, is_causal=True, scale=scale)
    ref = ref.transpose(1, 2).reshape(B * L, H, dv).numpy()
    np.testing.assert_allclose(out, ref, rtol=1e-11, atol=1e-12)


def test_attention_special_cases():
    q, k, v = _mha_case(L=10, seed=2)
    # one selected key -> its value row
    idx = np.full((10, 4), -1, np.int32)
    idx[:, 0] = 3
    out = oracle.sparse_attn(q.numpy(), k.numpy(), idx, 0.3, v=v.numpy())
    for h in range(2):
        np.testing.assert_allclose(out[:, h, :], np.broadcast_to(v[0, 3, h].double().numpy(), (10, 16)), rtol=0, atol=0)
    # q = 0 -> uniform weights -> mean of the selected value rows
    idx2 = np.array([[1, 4, 7, -1]] * 10, np.int32)
    out0 = oracle.sparse_attn(np.zeros_like(q.numpy()), k.numpy(), idx2, 0.3, v=v.numpy())
    mean = v[0, [1, 4, 7]].double().mean(0).numpy()       # [KVH, dv]
    for h in range(2):
        np.testing.assert_allclose(out0[:, h, :], np.broadcast_to(mean[h], (10, 16)), rtol=1e-14, atol=1e-15)
    # nothing selected -> zeros and lse = -inf
    idx3 = np.full((10, 4), -1, np.int32)
    out3, lse3 = oracle.sparse_attn(q.numpy(), k.numpy(), idx3, 0.3, v=v.numpy(), want_lse=True)
    assert np.all(out3 == 0) and np.all(np.isneginf(lse3))


def test_attention_sparse_equals_additive_mask_dense():
    """The port's additive-mask form and the index-driven form agree (DSA item 2)."""
    q, k, v = _mha_case(L=32, seed=7)
    g = np.random.default_rng(7)
    L, kk = 32, 8
    idx = np.full((L, kk), -1, np.int32)
    for t in range(L):
        sel = np.sort(g.choice(t + 1, size=min(kk, t + 1), replace=False))
        idx[t, : sel.size] = sel
    sp = oracle.sparse_attn(q.numpy(), k.numpy(), idx, 0.25, v=v.numpy())
    de = oracle.dense_masked_attn(q.numpy(), k.numpy(), idx, [0], 0.25, v=v.numpy())
    np.testing.assert_allclose(sp, de, rtol=1e-12, atol=1e-13)


def test_attention_gqa_head_grouping():
    """H heads over KVH kv heads: head h reads kv head h // (H // KVH)."""
    q, k, v = _mha_case(L=12, H=4, KVH=2, seed=8)
    idx = np.tile(np.arange(12, dtype=np.int32), (12, 1))
    idx = np.where(idx <= np.arange(12)[:, None], idx, -1).astype(np.int32)
    out = oracle.sparse_attn(q.numpy(), k.numpy(), idx, 0.25, v=v.numpy())
    kr = k.double().repeat_interleave(2, dim=2)
    vr = v.double().repeat_interleave(2, dim=2)
    ref = F.scaled_dot_product_attention(q.double().transpose(1, 2), kr.transpose(1, 2), vr.transpose(1, 2),
                                         is_causal=True, scale=0.25).transpose(1, 2)[0].numpy()
    np.testing.assert_allclose(out, ref, rtol=1e-11, atol=1e-12)


# ------------------------------------------------------------------ configs --

def test_workload_shapes_follow_config_defaults():
    cfg = json.load(open(os.path.join(GOLDEN, "deepseek_v32_config.json")))
    for name in ("decode32k", "prefill8k", "prefill64k", "decode128k"):
        wl = workloads.get(name)
        assert wl.topk == cfg["index_topk"]
        assert wl.idx_dim == cfg["index_head_dim"]
        assert wl.idx_heads == cfg["index_n_heads"]
        assert wl.heads == cfg["num_attention_heads"]
        assert wl.d_qk == cfg["kv_lora_rank"] + cfg["qk_rope_head_dim"]
        assert wl.d_v == cfg["kv_lora_rank"]
        assert wl.s_max <= cfg["max_position_embeddings"]
        assert wl.sm_scale == pytest.approx(1 / math.sqrt(cfg["qk_nope_head_dim"] + cfg["qk_rope_head_dim"]))


def test_tiny_workload_end_to_end_on_oracle():
    """The composition on the tiny workload: selected sets are causal, sized
    min(k, p+1), and attention over them equals the masked dense form."""
    wl = workloads.get("tiny")
    t = workloads.make_inputs(wl, "cpu", seed=0)
    n = {k: workloads.to_numpy(v) for k, v in t.items()}
    sc = oracle.indexer_scores(n["q_idx"], n["k_idx"], n["w"], n["ctx_len"], n["q_pos0"])
    pos = np.arange(wl.n_q, dtype=np.int32)
    idx = oracle.topk(np.where(np.isfinite(sc), sc, -np.inf).astype(np.float32), pos, wl.topk)
    cnt = (idx >= 0).sum(1)
    np.testing.assert_array_equal(cnt, np.minimum(wl.topk, pos + 1))
    assert np.all(idx.max(1) <= pos)
    out = oracle.sparse_attn(n["q"], n["kv"], idx, wl.sm_scale, v=n["v"])
    de = oracle.dense_masked_attn(n["q"], n["kv"], idx, n["q_pos0"], wl.sm_scale, v=n["v"])
    np.testing.assert_allclose(out, de, rtol=1e-12, atol=1e-13)


# ------------------------------------------------------------- cache append --

def _append_case(seed, B=3, s_max=16, n=5, D=128, Dkv=40):
    g = np.random.default_rng(seed)
    k_cache = g.integers(0, 2**16, size=(B, s_max, D)).astype(np.uint16)
    kv_cache = g.integers(0, 2**16, size=(B, s_max, Dkv)).astype(np.uint16)
    k_new = _bf16_bits(torch.from_numpy(g.standard_normal((B, n, D)).astype(np.float32) / 8))
    kv_new = g.integers(0, 2**16, size=(B, n, Dkv)).astype(np.uint16)
    return k_cache, kv_cache, k_new, kv_new


def test_cache_append_places_rows_and_leaves_the_rest():
    """Token i of sequence b lands in row pos[b] + i; every other row, and
    tokens whose row falls outside [0, s_max), change nothing."""
    k_cache, kv_cache, k_new, kv_new = _append_case(1)
    pos = np.array([3, 0, 13], np.int32)  # sequence 2: rows 13..17, only 13..15 exist
    kc, _, kvc, _ = oracle.cache_append(k_cache, kv_cache, k_new, kv_new, pos)
    for b in range(3):
        for r in range(16):
            i = r - pos[b]
            if 0 <= i < 5:
                np.testing.assert_array_equal(kc[b, r], k_new[b, i])
                np.testing.assert_array_equal(kvc[b, r], kv_new[b, i])
            else:
                np.testing.assert_array_equal(kc[b, r], k_cache[b, r])
                np.testing.assert_array_equal(kvc[b, r], kv_cache[b, r])
    neg = np.array([-2, 0, 0], np.int32)  # rows -2, -1 skipped, 0..2 written
    kc, _, _, _ = oracle.cache_append(k_cache, kv_cache, k_new, kv_new, neg)
    np.testing.assert_array_equal(kc[0, :3], k_new[0, 2:])
    np.testing.assert_array_equal(kc[0, 3:], k_cache[0, 3:])


def test_cache_append_fp8_round_trip_within_e4m3_bound():
    """E4M3 cache: decoding the codes, scaling and rotating back (H is its own
    inverse) recovers each key within the quantisation bound: every rotated
    element within 2^-4 relative or 2^-10 sigma absolute."""
    k_cache, kv_cache, k_new, kv_new = _append_case(2)
    codes0 = np.zeros(k_cache.shape, np.uint8)
    sc0 = np.zeros(k_cache.shape[:2], np.float32)
    pos = np.array([0, 4, 9], np.int32)
    kc, ks, _, _ = oracle.cache_append(codes0, kv_cache, k_new, kv_new, pos, k_scale=sc0)
    kf = torch.from_numpy(k_new.view(np.int16)).view(torch.bfloat16).float().numpy().astype(np.float64)
    for b in range(3):
        for i in range(5):
            r = pos[b] + i
            y = oracle.hadamard(kf[b, i])
            yq = oracle.e4m3_decode(kc[b, r]) * np.float64(ks[b, r])
            assert np.all(np.abs(yq - y) <= 2.0**-4 * np.abs(y) + 2.0**-10 * ks[b, r] + 1e-12)
            back = oracle.hadamard(yq)
            assert np.linalg.norm(back - kf[b, i]) <= 2.0**-4 * np.linalg.norm(kf[b, i]) + 1e-6
            assert ks[b, r] == np.float32(np.abs(y).max() / 448.0)


def test_cache_append_then_score_equals_scoring_the_full_keys():
    """Appending a sequence's keys one step at a time and scoring gives the
    scores of the whole key array (bf16 path, bit for bit), and the FP8 cache
    equals quantising the whole key array at once."""
    g = np.random.default_rng(3)
    B, S, H, D = 2, 24, 4, 128
    k_full = _bf16_bits(torch.from_numpy(g.standard_normal((B, S, D)).astype(np.float32) / 11))
    q = _bf16_bits(torch.from_numpy(g.standard_normal((B, 1, H, D)).astype(np.float32) / 11))
    w = g.standard_normal((B, 1, H)).astype(np.float32)
    k_cache = np.zeros((B, S, D), np.uint16)
    kv_cache = np.zeros((B, S, 8), np.uint16)
    c8 = np.zeros((B, S, D), np.uint8)
    s8 = np.zeros((B, S), np.float32)
    for t0, n in ((0, 10), (10, 1), (11, 13)):  # a prefill chunk, a decode step, the rest
        kn = np.ascontiguousarray(k_full[:, t0:t0 + n])
        kvn = np.zeros((B, n, 8), np.uint16)
        pos = np.full(B, t0, np.int32)
        k_cache, _, kv_cache, _ = oracle.cache_append(k_cache, kv_cache, kn, kvn, pos)
        c8, s8, _, _ = oracle.cache_append(c8, kv_cache, kn, kvn, pos, k_scale=s8)
    ctx, pos0 = [S, S], [S - 1, S - 1]
    np.testing.assert_array_equal(oracle.indexer_scores(q, k_cache, w, ctx, pos0),
                                  oracle.indexer_scores(q, k_full, w, ctx, pos0))
    cf, sf, _ = oracle.hadamard_quant(k_full)
    np.testing.assert_array_equal(c8, cf)
    np.testing.assert_array_equal(s8, sf)


# -------------------------------------------------------------- projections --

def test_linear_matches_blas_on_bf16_inputs():
    """Y = X W^T: the oracle's loop sum against a BLAS matrix product of the
    exactly widened bf16 values, on the wq_b inner size (q_lora_rank 1536)
    and the hidden size (7168)."""
    g = torch.Generator().manual_seed(3)
    for K, N in ((1536, 96), (7168, 40)):
        x = torch.randn(13, K, generator=g) / math.sqrt(K)
        w = torch.randn(N, K, generator=g)
        xb, wb = _bf16_bits(x), _bf16_bits(w)
        xf = x.to(torch.bfloat16).double().numpy()
        wf = w.to(torch.bfloat16).double().numpy()
        np.testing.assert_allclose(oracle.linear(xb, wb), xf @ wf.T, rtol=1e-12, atol=1e-12)


def test_linear_one_hot_rows_select_columns_and_orientation():
    """A one-hot row n of W (1 at column c_n) makes output column n equal to
    input column c_n exactly; a transposed operand or swapped index fails."""
    g = np.random.default_rng(4)
    M, K, N = 9, 64, 5
    x = g.standard_normal((M, K)).astype(np.float32)
    cols = [3, 0, 63, 17, 17]
    w = np.zeros((N, K), dtype=np.float32)
    for n, c in enumerate(cols):
        w[n, c] = 1.0
    y = oracle.linear(x, w)
    for n, c in enumerate(cols):
        np.testing.assert_array_equal(y[:, n], x[:, c].astype(np.float64))
    # rows of X stay rows of Y: leading shape kept, rows independent
    y3 = oracle.linear(x.reshape(3, 3, K), w)
    np.testing.assert_array_equal(y3.reshape(M, N), y)


def test_linear_is_linear_in_both_operands():
    g = np.random.default_rng(5)
    x1, x2 = g.standard_normal((2, 6, 32)).astype(np.float32)
    w = g.standard_normal((7, 32)).astype(np.float32)
    a = oracle.linear(x1, w) + oracle.linear(x2, w)
    np.testing.assert_allclose(oracle.linear((x1 + x2).astype(np.float32), w), a, rtol=1e-6, atol=1e-5)
    np.testing.assert_allclose(oracle.linear(x1, (-w).astype(np.float32)), -oracle.linear(x1, w), rtol=0, atol=0)
