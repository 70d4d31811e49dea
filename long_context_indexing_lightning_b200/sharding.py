"""Prefill of one long sequence split across GPUs by query rows.

DeepSeek-V3.2 model doc (Transformers), section "DeepSeek Sparse Attention
(DSA)": each query scores every earlier key of the indexer's own key cache
(item 1) and attends only over its own index_topk selection (item 2), so once
the caches hold the sequence, query rows are independent.  A prefill then
splits by query rows, one process per GPU:

  1. each rank writes an equal share of the new tokens' rows into its copy of
     the index-key and latent caches (``cache_append``: the tokens are the
     prefill's own queries),
  2. one all-gather per cache tensor gives every rank all the new rows
     (``gather_cache_rows``; over NVLink / NVSwitch with NCCL),
  3. each rank runs the layer step on its own contiguous range of query rows
     (``forward`` with ``rank_shape``: q_pos0 moved to the range's first
     position); ranges come from ``balanced_row_ranges``, which evens out the
     causal cost (a query at position p scores p + 1 keys and attends over
     min(p + 1, index_topk) rows).

Scores, selections and outputs never cross ranks.  Decode needs none of this:
it splits by sequence with no collective at all.  These functions are host
plumbing around the library's entry points; every step of the path runs in
its kernels.
"""
import math

import torch
import torch.distributed as dist

# Time of one attention row relative to scoring one (query, key) pair plus its
# top-k share, from the 64K-token prefill on one B200: indexer + top-k
# 59 ms over 2.15e9 causal pairs, attention 85 ms over 1.32e8 selected rows.
ATTN_ROW_COST = 23.0


def row_cost(p, topk, attn_row_cost=ATTN_ROW_COST):
    """Relative cost of the query at position p (0-based)."""
    return (p + 1) + attn_row_cost * min(p + 1, topk)


def _cum_cost(t, pos0, topk, a):
    """Sum of row_cost over the queries at positions pos0 .. pos0 + t - 1."""
    def tri(n):  # sum of (p + 1) for p < n
        return n * (n + 1) // 2

    def capped(n):  # sum of min(p + 1, topk) for p < n
        m = min(n, topk)
        return tri(m) + (n - m) * topk

    lo, hi = pos0, pos0 + t
    return (tri(hi) - tri(lo)) + a * (capped(hi) - capped(lo))


def balanced_row_ranges(n_q, world, pos0=0, topk=2048, attn_row_cost=ATTN_ROW_COST):
    """Split query rows [0, n_q) (positions pos0 ..) into `world` contiguous
    ranges [start, stop) of near-equal causal cost, in rank order.  Range r
    ends at the first row where the running cost reaches (r + 1) / world of
    the total, so every range's cost is within one row's cost of the even
    share.  Ranges may be empty when n_q < world."""
    if n_q < 0 or world < 1:
        raise ValueError("n_q >= 0 and world >= 1")
    total = _cum_cost(n_q, pos0, topk, attn_row_cost)
    bounds = [0]
    for r in range(1, world):
        target = total * r / world
        lo, hi = bounds[-1], n_q  # first t in [lo, hi] with cum(t) >= target
        while lo < hi:
            mid = (lo + hi) // 2
            if _cum_cost(mid, pos0, topk, attn_row_cost) >= target:
                hi = mid
            else:
                lo = mid + 1
        bounds.append(lo)
    bounds.append(n_q)
    return [(bounds[r], bounds[r + 1]) for r in range(world)]


def append_share(n_new, world, rank):
    """Token range [start, stop) (relative to the first new token) that `rank`
    appends: equal shares of ceil(n_new / world) rows, the last one short."""
    c = math.ceil(n_new / world) if n_new > 0 else 0
    start = min(rank * c, n_new)
    return start, min(start + c, n_new)


def rank_shape(shape, start, stop):
    """The shape of one rank's part of the step: its stop - start query rows."""
    return shape.replace(n_q=stop - start)


def gather_cache_rows(cache, b, row0, n_new, group=None):
    """All-gather the new rows [row0, row0 + n_new) of sequence b of `cache`
    (shape [B, s_max, ...]) across the ranks of `group`, where each rank has
    written its append_share of them.  One collective, in place: rank r's
    ceil(n_new / world) rows are its chunk of the gathered range.  The last
    chunk may run past row0 + n_new: those rows (beyond the new context) take
    whatever the last rank holds there, so the gathered range must fit in
    s_max."""
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    if world == 1 or n_new == 0:
        return cache
    c = math.ceil(n_new / world)
    if row0 < 0 or row0 + world * c > cache.shape[1]:
        raise ValueError(f"rows [{row0}, {row0 + world * c}) of the gathered range do not fit in "
                         f"s_max = {cache.shape[1]}")
    seq = cache[b]
    if not seq.is_contiguous():
        raise ValueError("cache rows of one sequence must be contiguous")
    out = seq[row0:row0 + world * c]
    dist.all_gather_into_tensor(out, out[rank * c:(rank + 1) * c], group=group)
    return cache


def prefill_rank(dsa, shape, pos0, rows, k_new, kv_new, k_cache, kv_cache, q_idx, w, q, ctx_len, k_scale=None,
                 group=None, **forward_kw):
    """One rank's part of a sharded prefill of one sequence; ``dsa`` is the
    library binding and everything runs on the current stream (the
    collectives wait for it).

    shape: the whole prefill (batch 1, n_q = n_new new tokens at positions
        pos0 .. pos0 + n_new - 1).
    k_new [1, a, idx_dim], kv_new [1, a, d_qk]: this rank's append_share of
        the new tokens (a rows, bf16 keys; e4m3 caches quantise them).
    k_cache, kv_cache (and k_scale): the sequence's caches, [1, s_max, ...].
    q_idx, w, q: this rank's query rows [rows[0], rows[1]) of
        balanced_row_ranges; ctx_len: [1] int32 device, pos0 + n_new.
    Returns this rank's attention output, [1, rows[1] - rows[0], H, d_v]."""
    if shape.batch != 1:
        raise ValueError("prefill_rank takes one sequence (shape.batch == 1)")
    world = dist.get_world_size(group) if dist.is_initialized() else 1
    rank = dist.get_rank(group) if dist.is_initialized() else 0
    n_new = shape.n_q
    a0, a1 = append_share(n_new, world, rank)
    if a1 > a0:
        pos = torch.full((1,), pos0 + a0, dtype=torch.int32, device=k_cache.device)
        dsa.cache_append(shape.replace(n_q=1), k_new, kv_new, pos, k_cache, kv_cache, k_scale=k_scale)
    if world > 1:
        gather_cache_rows(k_cache, 0, pos0, n_new, group)
        if k_scale is not None:
            gather_cache_rows(k_scale, 0, pos0, n_new, group)
        gather_cache_rows(kv_cache, 0, pos0, n_new, group)
    r0, r1 = rows
    q_pos0 = torch.full((1,), pos0 + r0, dtype=torch.int32, device=k_cache.device)
    return dsa.forward(rank_shape(shape, r0, r1), q_idx, k_cache, w, q, kv_cache, ctx_len, q_pos0,
                       k_scale=k_scale, **forward_kw)
