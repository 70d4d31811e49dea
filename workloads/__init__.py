"""Seeded synthetic workloads for the DSA layer step.

This module only draws random inputs and names shapes; it holds none of the
method's arithmetic, so both the CUDA path's tests/benchmark and the CPU
oracle may take their inputs from it.

Shapes follow the DeepSeek-V3.2 configuration (Transformers model doc,
section DeepseekV32Config): index_n_heads 64, index_head_dim 128,
index_topk 2048, num_attention_heads 128, kv_lora_rank 512,
qk_rope_head_dim 64 (latent row = 512 + 64 = 576 columns, value = the first
512).  The pages give no value distributions; the recipe below is ours:
standard normal draws in fp32, scaled, then rounded to bf16 (RNE).
Draw order is fixed: q_idx, k_idx, w, q, kv (then v for the MHA case).
"""
from dataclasses import dataclass, field, replace
import math

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    n_q: int            # queries per sequence (1 = decode)
    s_max: int          # cache capacity == ctx_len for the named workloads
    idx_heads: int
    idx_dim: int
    topk: int
    heads: int
    d_qk: int
    d_v: int
    kv_heads: int       # 1 = absorbed MLA (one shared latent row, V = its first d_v columns)
    dtype: str          # "bf16" or "f32" storage of q/k inputs
    q_idx_std: float
    k_idx_std: float
    w_std: float
    q_std: float
    kv_std: float
    sm_scale: float
    idx_scale: float = 1.0
    decode: bool = False  # query sits at ctx_len-1 (its own key is already cached)
    idx_fp8: bool = False
    idx_rescore: int = 0  # e4m3 indexer: extra FP8 candidates re-scored from the bf16 keys
    ctx_len: tuple = field(default=None)  # per-sequence lengths; None = all s_max

    def lengths(self):
        return list(self.ctx_len) if self.ctx_len is not None else [self.s_max] * self.batch

    def positions0(self):
        if self.decode:
            return [L - self.n_q for L in self.lengths()]
        return [0] * self.batch


_MLA = dict(idx_heads=64, idx_dim=128, topk=2048, heads=128, d_qk=576, d_v=512, kv_heads=1,
            dtype="bf16", q_idx_std=1 / math.sqrt(128), k_idx_std=1 / math.sqrt(128), w_std=1 / 8,
            q_std=1.0, kv_std=1.0, sm_scale=1 / math.sqrt(192))

WORKLOADS = {
    # tiny causal prefill: fp32, MHA with 2 heads (separate k and v per head)
    "tiny": Workload("tiny", batch=1, n_q=256, s_max=256, idx_heads=4, idx_dim=32, topk=16, heads=2,
                     d_qk=32, d_v=32, kv_heads=2, dtype="f32", q_idx_std=1 / math.sqrt(32),
                     k_idx_std=1 / math.sqrt(32), w_std=0.5, q_std=1 / math.sqrt(32),
                     kv_std=1 / math.sqrt(32), sm_scale=1 / math.sqrt(32)),
    "decode32k": Workload("decode32k", batch=8, n_q=1, s_max=32768, decode=True, **_MLA),
    "prefill8k": Workload("prefill8k", batch=1, n_q=8192, s_max=8192, **_MLA),
    "prefill64k": Workload("prefill64k", batch=1, n_q=65536, s_max=65536, **_MLA),
    "decode128k": Workload("decode128k", batch=32, n_q=1, s_max=131072, decode=True, **_MLA),
    "decode128k_fp8": Workload("decode128k_fp8", batch=32, n_q=1, s_max=131072, decode=True,
                               idx_fp8=True, idx_rescore=1024, **_MLA),
}


def get(name: str, **overrides) -> Workload:
    wl = WORKLOADS[name]
    return replace(wl, **overrides) if overrides else wl


_DRAW = 1 << 26  # elements per fp32 draw (bounds the temporary buffer)


def _randn_into(out: torch.Tensor, gen: torch.Generator, std: float):
    """Fill ``out`` with N(0, std^2) drawn in fp32, in consecutive pieces of at
    most 2^26 elements (one leading-axis slice at a time)."""
    flat = out.view(out.shape[0], -1)
    for i in range(flat.shape[0]):
        row = flat[i]
        for j in range(0, row.numel(), _DRAW):
            n = min(_DRAW, row.numel() - j)
            x = torch.randn(n, generator=gen, device=out.device, dtype=torch.float32)
            row[j:j + n].copy_(x.mul_(std))


def make_inputs(wl: Workload, device="cpu", seed: int = 0, attention: bool = True):
    """Draw one batch of inputs for ``wl`` on ``device`` with a seeded generator.

    Returns a dict of tensors:
      q_idx [B, n_q, H_I, D_I], k_idx [B, s_max, D_I], w [B, n_q, H_I] fp32,
      q [B, n_q, H, d_qk], kv [B, s_max, KVH, d_qk] (KVH = 1 squeezed: [B, s_max, d_qk]),
      v [B, s_max, KVH, d_v] (MHA only), ctx_len [B] int32, q_pos0 [B] int32.
    """
    dt = torch.bfloat16 if wl.dtype == "bf16" else torch.float32
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    B = wl.batch
    t = {}
    t["q_idx"] = torch.empty(B, wl.n_q, wl.idx_heads, wl.idx_dim, dtype=dt, device=device)
    _randn_into(t["q_idx"], gen, wl.q_idx_std)
    t["k_idx"] = torch.empty(B, wl.s_max, wl.idx_dim, dtype=dt, device=device)
    _randn_into(t["k_idx"], gen, wl.k_idx_std)
    t["w"] = torch.empty(B, wl.n_q, wl.idx_heads, dtype=torch.float32, device=device)
    _randn_into(t["w"], gen, wl.w_std)
    if attention:
        t["q"] = torch.empty(B, wl.n_q, wl.heads, wl.d_qk, dtype=dt, device=device)
        _randn_into(t["q"], gen, wl.q_std)
        if wl.kv_heads == 1:
            t["kv"] = torch.empty(B, wl.s_max, wl.d_qk, dtype=dt, device=device)
        else:
            t["kv"] = torch.empty(B, wl.s_max, wl.kv_heads, wl.d_qk, dtype=dt, device=device)
        _randn_into(t["kv"], gen, wl.kv_std)
        if wl.kv_heads > 1:
            t["v"] = torch.empty(B, wl.s_max, wl.kv_heads, wl.d_v, dtype=dt, device=device)
            _randn_into(t["v"], gen, wl.kv_std)
    t["ctx_len"] = torch.tensor(wl.lengths(), dtype=torch.int32, device=device)
    t["q_pos0"] = torch.tensor(wl.positions0(), dtype=torch.int32, device=device)
    return t


def to_numpy(x: torch.Tensor):
    """Host numpy view of a tensor in its stored type (bf16 -> uint16 bits)."""
    x = x.detach().contiguous().cpu()
    if x.dtype == torch.bfloat16:
        return x.view(torch.int16).numpy().view("uint16")
    return x.numpy()


def sample_rows(n_q: int, count: int, seed: int = 1, extra=()):
    """Query rows to check on a large prefill: ``count`` drawn uniformly without
    replacement (numpy PCG64), plus the listed rows; sorted, unique."""
    import numpy as np
    rng = np.random.Generator(np.random.PCG64(seed))
    pick = rng.choice(n_q, size=min(count, n_q), replace=False)
    rows = set(int(r) for r in pick) | set(int(r) for r in extra if 0 <= r < n_q)
    return sorted(rows)
