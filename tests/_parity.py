"""Comparison rules shared by the GPU parity tests.

Tolerances:
  * indexer scores: |g - o| <= 1e-3 * (|o| + rms(o_row)), rms over the row's
    finite entries; -inf must match -inf exactly.
  * top-k on identical fp32 scores: bit-exact index lists.
  * top-k on end-to-end scores: the sets agree except for indices whose
    oracle score is within 1e-3 * (|tau| + rms(o_row)) of the oracle's k-th
    score tau; set sizes are equal.
  * attention (bf16 in/out): max |g - o| <= 2e-2 against the fp64 oracle.
"""
import numpy as np

SCORE_RTOL = 1e-3
ATTN_ATOL_BF16 = 2e-2


def rms_finite(row):
    f = row[np.isfinite(row)]
    return float(np.sqrt(np.mean(f * f))) if f.size else 0.0


def check_scores(gpu, ora, valid_len, rtol=SCORE_RTOL, what="scores"):
    """gpu: fp32 [nrows, >= S]; ora: fp64 [nrows, S]; valid_len[r]: columns compared."""
    worst = 0.0
    for r in range(ora.shape[0]):
        L = int(valid_len[r])
        g = gpu[r, :L].astype(np.float64)
        o = ora[r, :L]
        ninf = np.isneginf(o)
        assert np.array_equal(np.isneginf(g), ninf), f"{what}: -inf pattern differs in row {r}"
        fin = ~ninf
        tol = rtol * (np.abs(o[fin]) + rms_finite(o))
        err = np.abs(g[fin] - o[fin])
        bad = err > tol
        assert not bad.any(), (f"{what}: row {r}: {int(bad.sum())} entries out of tolerance, "
                               f"first at {int(np.nonzero(fin)[0][np.argmax(bad)])}: gpu {g[fin][bad][0]!r} "
                               f"oracle {o[fin][bad][0]!r}")
        if tol.size:
            worst = max(worst, float((err / np.maximum(tol, 1e-300)).max()))
    return worst


def check_topk_near_ties(gpu_idx, ora_idx, ora_scores, k, rtol=SCORE_RTOL):
    """End-to-end rule: sets equal up to swaps at the k-th score."""
    swaps = 0
    for r in range(ora_idx.shape[0]):
        g = set(int(x) for x in gpu_idx[r] if x >= 0)
        o = set(int(x) for x in ora_idx[r] if x >= 0)
        assert len(g) == len(o), f"row {r}: set sizes {len(g)} vs {len(o)}"
        diff = g ^ o
        if not diff:
            continue
        row = ora_scores[r]
        sel = np.array(sorted(o))
        tau = float(np.min(row[sel]))
        tol = rtol * (abs(tau) + rms_finite(row))
        for i in diff:
            assert abs(row[i] - tau) <= tol, f"row {r}: index {i} score {row[i]} vs k-th {tau} (tol {tol})"
        swaps += len(diff) // 2
    return swaps


def check_idx_valid(idx, pos, k):
    """Ascending, causal, unique, count = min(k, pos+1), -1 padding."""
    for r in range(idx.shape[0]):
        row = idx[r]
        n = min(k, int(pos[r]) + 1)
        sel = row[:n]
        assert np.all(row[n:] == -1), f"row {r}: padding"
        assert np.all(sel >= 0) and np.all(sel <= pos[r]), f"row {r}: causal"
        assert np.all(np.diff(sel) > 0), f"row {r}: ascending/unique"


def bf16_bits_to_f64(bits):
    return (np.asarray(bits).astype(np.uint32) << 16).view(np.float32).astype(np.float64)
