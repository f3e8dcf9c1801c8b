"""Comparison rules shared by the parity tests.

Index rule: the GPU's selected set must equal the oracle's, except for keys
whose oracle score lies within REL_TIE (relative) of the oracle's k-th score:
such near-ties may be swapped in or out, because the GPU ranks fp32 scores
and the oracle ranks exact (double) ones.

Attention rule (computed on the oracle's indices): max-abs error 2e-2 for
bf16 outputs, 1e-4 for fp32 outputs.
"""
import numpy as np

REL_TIE = 1e-3
ATOL_OUT = {"bf16": 2e-2, "fp32": 1e-4}
ATOL_LSE = {"bf16": 2e-2, "fp32": 1e-4}


def check_index_sets(gpu_idx: np.ndarray, oracle_scores: np.ndarray, oracle_idx: np.ndarray, k: int,
                     rel: float = REL_TIE):
    """gpu_idx, oracle_idx: [n, k] int (-1 = unused); oracle_scores [n, L]
    double.  Returns the number of near-tie swaps; raises AssertionError on a
    mismatch outside the band."""
    swaps = 0
    for r in range(gpu_idx.shape[0]):
        g = set(int(x) for x in gpu_idx[r] if x >= 0)
        o = set(int(x) for x in oracle_idx[r] if x >= 0)
        assert len(g) == len([x for x in gpu_idx[r] if x >= 0]), f"row {r}: duplicate indices"
        assert len(g) == len(o), f"row {r}: {len(g)} selected, oracle {len(o)}"
        if g == o:
            continue
        kth = min(oracle_scores[r, s] for s in o)
        band = rel * abs(kth)
        for s in g ^ o:
            assert abs(oracle_scores[r, s] - kth) <= band, (
                f"row {r}: key {s} (score {oracle_scores[r, s]!r}) differs from the oracle set outside the "
                f"near-tie band around the k-th score {kth!r}")
        swaps += len(g - o)
    return swaps


def check_sorted_unique(idx: np.ndarray, n_visible: np.ndarray):
    """GPU contract: ascending positions, then -1 tail; count = min(k, n)."""
    k = idx.shape[1]
    for r in range(idx.shape[0]):
        sel = idx[r][idx[r] >= 0]
        want = min(k, int(n_visible[r]))
        assert len(sel) == want, f"row {r}: {len(sel)} selected, expected {want}"
        assert np.all(idx[r][want:] == -1), f"row {r}: -1 tail broken"
        assert np.all(np.diff(sel) > 0), f"row {r}: not strictly ascending"
        assert sel.size == 0 or (sel[0] >= 0 and sel[-1] < n_visible[r]), f"row {r}: position out of range"
