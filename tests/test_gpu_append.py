"""GPU parity of the cache append (dsa_cache_append) against the oracle.

The indexer keeps its own per-token key cache beside the K/V cache and it is
updated before the step scores (DeepSeek-V3.2 model doc, section "DeepSeek
Sparse Attention (DSA)"); the reference indexer's cache is FP8 after the
Hadamard rotation.  Copies must be bit-exact; e4m3 codes must equal the
oracle's except where the oracle's unrounded quotient sits on a rounding
boundary (the same rule as the query quantiser's test).
"""
import numpy as np
import pytest
import torch

import long_context_indexing_lightning_b200 as dsa
import oracle
import workloads
from long_context_indexing_lightning_b200 import build

from test_gpu_parity import _codes_ok

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


def _rand_bf16(g, *shape, scale=1.0):
    return (torch.randn(*shape, generator=g, device=DEV) * scale).to(torch.bfloat16)


def _case(B, s_max, n, fp8, seed, d_qk=576, pos=None):
    g = torch.Generator(device=DEV).manual_seed(seed)
    k_new = _rand_bf16(g, B, n, 128, scale=128 ** -0.5)
    kv_new = _rand_bf16(g, B, n, d_qk)
    kv_cache = _rand_bf16(g, B, s_max, d_qk)
    if fp8:
        k_cache = torch.randint(0, 255, (B, s_max, 128), generator=g, device=DEV, dtype=torch.int32).to(torch.uint8)
        k_scale = torch.rand(B, s_max, generator=g, device=DEV)
    else:
        k_cache = _rand_bf16(g, B, s_max, 128)
        k_scale = None
    if pos is None:
        pos = torch.randint(0, s_max - n + 1, (B,), generator=g, device=DEV, dtype=torch.int32)
    else:
        pos = torch.tensor(pos, dtype=torch.int32, device=DEV)
    return k_new, kv_new, k_cache, k_scale, kv_cache, pos


def _check(B, s_max, n, fp8, seed, pos=None):
    k_new, kv_new, k_cache, k_scale, kv_cache, pos = _case(B, s_max, n, fp8, seed, pos=pos)
    before = {k: H(v) for k, v in dict(k_new=k_new, kv_new=kv_new, k_cache=k_cache, kv_cache=kv_cache,
                                         pos=pos).items()}
    ks_before = H(k_scale) if fp8 else None
    shape = dsa.make_shape(B, 1, s_max, idx_dtype=dsa.DSA_E4M3 if fp8 else dsa.DSA_BF16)
    dsa.cache_append(shape, k_new, kv_new, pos, k_cache, kv_cache, k_scale=k_scale)
    torch.cuda.synchronize()
    ok, ks, okv, _ = oracle.cache_append(before["k_cache"], before["kv_cache"], before["k_new"], before["kv_new"],
                                         before["pos"], k_scale=ks_before)
    np.testing.assert_array_equal(H(kv_cache), okv)
    if fp8:
        _, _, quot = oracle.hadamard_quant(before["k_new"])
        # the unrounded quotient of every cache row (rows not written keep no quotient: codes must be equal)
        qfull = np.zeros(ok.shape, np.float64)
        for b in range(B):
            for i in range(n):
                r = int(before["pos"][b]) + i
                if 0 <= r < s_max:
                    qfull[b, r] = quot[b, i]
        assert _codes_ok(H(k_cache), ok, qfull) <= 8 * B * n
        np.testing.assert_allclose(H(k_scale), ks, rtol=2e-6, atol=0)
    else:
        np.testing.assert_array_equal(H(k_cache), ok)
    return pos


@pytest.mark.parametrize("fp8", [False, True])
def test_append_decode_step_matches_oracle(fp8):
    """One new token per sequence (decode), 32 sequences, bf16 / e4m3 key cache."""
    _check(32, 4096, 1, fp8, seed=1)


@pytest.mark.parametrize("fp8", [False, True])
def test_append_prefill_chunk_matches_oracle(fp8):
    """A 4096-token prefill chunk into a 65536-row cache."""
    _check(1, 65536, 4096, fp8, seed=2, pos=[61000])


def test_append_out_of_range_rows_are_skipped_and_flagged():
    dsa.get_error(clear=True)
    _check(3, 64, 8, False, seed=3, pos=[60, -3, 10])  # rows 64..67 and -3..-1 do not exist
    rc, word = dsa.get_error(clear=True)
    assert rc == 6 and word & 2  # DSA_ERR_BAD_INDEX


def test_append_separate_v_fp32_form():
    """The fp32 MHA form (kv_heads 2, separate k and v rows) copies both."""
    g = torch.Generator(device=DEV).manual_seed(4)
    B, s_max, n, KVH, d = 2, 40, 3, 2, 32
    k_new = torch.randn(B, n, 32, generator=g, device=DEV)
    kv_new = torch.randn(B, n, KVH, d, generator=g, device=DEV)
    v_new = torch.randn(B, n, KVH, d, generator=g, device=DEV)
    k_cache = torch.randn(B, s_max, 32, generator=g, device=DEV)
    kv_cache = torch.randn(B, s_max, KVH, d, generator=g, device=DEV)
    v_cache = torch.randn(B, s_max, KVH, d, generator=g, device=DEV)
    pos = torch.tensor([5, 38], dtype=torch.int32, device=DEV)  # the second runs off the end (row 40)
    hk, hkv, hv = H(k_cache), H(kv_cache), H(v_cache)
    shape = dsa.make_shape(B, 1, s_max, idx_heads=4, idx_dim=32, topk=16, heads=2, d_qk=d, d_v=d, kv_heads=KVH,
                           idx_dtype=dsa.DSA_F32, attn_dtype=dsa.DSA_F32)
    dsa.get_error(clear=True)
    dsa.cache_append(shape, k_new, kv_new, pos, k_cache, kv_cache, v_new=v_new, v_cache=v_cache)
    torch.cuda.synchronize()
    ok, _, okv, ov = oracle.cache_append(hk, hkv, H(k_new), H(kv_new), H(pos), v_cache=hv, v_new=H(v_new))
    np.testing.assert_array_equal(H(k_cache), ok)
    np.testing.assert_array_equal(H(kv_cache), okv)
    np.testing.assert_array_equal(H(v_cache), ov)
    rc, word = dsa.get_error(clear=True)
    assert rc == 6 and word & 2  # row 40 of sequence 1 does not exist


def test_append_then_forward_equals_forward_on_the_filled_cache():
    """Update before score: appending this step's token at ctx_len - 1 and
    running the step gives the output of the step on a cache that already
    held it (bit for bit)."""
    wl = workloads.get("decode32k", batch=4, s_max=8192)
    t = workloads.make_inputs(wl, DEV, seed=9)
    shape = dsa.shape_from_workload(wl)
    ref = dsa.forward(shape, t["q_idx"], t["k_idx"], t["w"], t["q"], t["kv"], t["ctx_len"], t["q_pos0"])
    last = (t["ctx_len"] - 1).to(torch.int32)
    b = torch.arange(wl.batch, device=DEV)
    k_new = t["k_idx"][b, last.long()].unsqueeze(1).contiguous()
    kv_new = t["kv"][b, last.long()].unsqueeze(1).contiguous()
    k_cache = t["k_idx"].clone()
    kv_cache = t["kv"].clone()
    k_cache[b, last.long()] = 0
    kv_cache[b, last.long()] = 0
    dsa.cache_append(shape, k_new, kv_new, last, k_cache, kv_cache)
    out = dsa.forward(shape, t["q_idx"], k_cache, t["w"], t["q"], kv_cache, t["ctx_len"], t["q_pos0"])
    torch.cuda.synchronize()
    assert torch.equal(out, ref)
