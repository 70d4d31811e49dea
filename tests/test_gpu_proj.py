"""GPU parity of the indexer projections (tensor-core GEMM) against the fp64
oracle: wq_b on the query latent and the fused key projection +
weights_proj on the hidden state, at the DeepSeek-V3.2 sizes (q_lora_rank
1536, hidden 7168, 64 index heads x 128), with token counts that leave a
ragged last 128-row tile.  Weights are seeded synthetic draws.

Tolerance: fp32 accumulation of K products then (bf16 outputs) one
round-to-nearest: |g - o| <= 2^-8 |o| + 1e-5 sqrt(K) rms(o) for bf16 outputs,
1e-5 (|o| + sqrt(K) rms(o)) / sqrt(K)... written out below per output type.
"""
import math

import numpy as np
import pytest
import torch

import long_context_indexing_lightning_b200 as dsa
import oracle
import workloads
from long_context_indexing_lightning_b200 import build

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


def _draw(shape, std, seed):
    g = torch.Generator(device=DEV).manual_seed(seed)
    return (torch.randn(*shape, generator=g, device=DEV) * std).to(torch.bfloat16)


def _check(got, want, K, bf16_out):
    got = got.astype(np.float64)
    rms = float(np.sqrt(np.mean(want * want)))
    # fp32 accumulation over K terms: a few units of 2^-24 times sqrt(K) of the row scale
    acc_tol = 8 * 2.0 ** -24 * math.sqrt(K) * rms
    tol = (2.0 ** -8 * np.abs(want) if bf16_out else 2.0 ** -22 * np.abs(want)) + acc_tol
    bad = np.abs(got - want) > tol
    assert not bad.any(), (int(bad.sum()), float(np.abs(got - want).max()))


@pytest.mark.parametrize("T", [1, 32, 300])
def test_proj_q_matches_oracle(T):
    shape = dsa.make_shape(1, 1, 1024)
    r = 1536
    x = _draw((T, r), 1.0, 40 + T)
    wq = _draw((64 * 128, r), 1 / math.sqrt(r), 41)
    q = dsa.indexer_proj_q(shape, x, wq)
    want = oracle.linear(H(x), H(wq))
    got = q.reshape(T, -1).float().cpu().numpy()
    _check(got, want, r, bf16_out=True)


@pytest.mark.parametrize("T", [1, 200])
def test_proj_kw_matches_oracle(T):
    shape = dsa.make_shape(1, 1, 1024)
    hidden = 7168
    x = _draw((T, hidden), 1.0, 50 + T)
    wkw = _draw((128 + 64, hidden), 1 / math.sqrt(hidden), 51)
    k_new, w = dsa.indexer_proj_kw(shape, x, wkw)
    want = oracle.linear(H(x), H(wkw))
    _check(k_new.float().cpu().numpy(), want[:, :128], hidden, bf16_out=True)
    _check(w.cpu().numpy(), want[:, 128:], hidden, bf16_out=False)


def test_projections_feed_the_step():
    """Projections -> cache append -> step, against the oracle run on the
    projections' own outputs (the step's parity is covered elsewhere; this
    checks the layouts the projections write are the ones the step reads)."""
    T, r, hidden = 700, 1536, 7168
    shape = dsa.make_shape(1, T, T, topk=256)
    lat = _draw((T, r), 1.0, 60)
    xh = _draw((T, hidden), 1.0, 61)
    wq = _draw((64 * 128, r), 1 / math.sqrt(r), 62)
    wkw = _draw((128 + 64, hidden), 1 / math.sqrt(hidden), 63)
    q_idx = dsa.indexer_proj_q(shape, lat, wq).reshape(1, T, 64, 128)
    k_new, w = dsa.indexer_proj_kw(shape, xh, wkw)
    ctx = torch.tensor([T], dtype=torch.int32, device=DEV)
    pos0 = torch.zeros(1, dtype=torch.int32, device=DEV)
    sc = dsa.indexer_scores(shape, q_idx, k_new.reshape(1, T, 128), w.reshape(1, T, 64), ctx, pos0)
    rows = [(0, t) for t in (0, 1, 255, 256, 511, 699)]
    o = oracle.indexer_scores(H(q_idx), H(k_new.reshape(1, T, 128)), H(w.reshape(1, T, 64)), H(ctx), H(pos0),
                              rows=rows)
    from _parity import check_scores
    g = sc.reshape(T, -1)[[t for _, t in rows]].cpu().numpy()
    check_scores(g, o, [T] * len(rows))
