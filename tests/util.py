"""Helpers shared by the tests: workload -> oracle arguments, tolerances, comparisons."""
from __future__ import annotations

import numpy as np

import oracle

# Parity bar for the output O (fp32 output), against the oracle's fp32 result.
O_MAX_ABS = 2e-3
O_MEAN_ABS = 2e-4

# (case, max-abs, mean-abs, P-code mismatches or None, codes compared) per parity check, printed
# in the terminal summary of the run (tests/conftest.py).
PARITY_STATS = []


def record_parity(case: str, max_abs: float, mean_abs: float, p_mismatch=None, p_total=None):
    PARITY_STATS.append((case, max_abs, mean_abs, p_mismatch, p_total))


def oracle_bias(w) -> "oracle.Bias":
    if w.bias_kind == 0 or w.bias is None:
        return oracle.Bias()
    return oracle.Bias(w.bias_kind, w.bias.float().numpy(), w.batch_stride, w.grid_h, w.grid_w,
                       w.table_h, w.table_w, w.n_prefix)


def oracle_qkv(w):
    return w.q.float().numpy(), w.k.float().numpy(), w.v.float().numpy()


def oracle_forward(w, rows=None, num_threads=0, softmax_scale=0.0):
    q, k, v = oracle_qkv(w)
    return oracle.get().attention_fwd(q, k, v, oracle_bias(w), softmax_scale=softmax_scale, block_c=128,
                                      num_threads=num_threads, rows=rows)


def oracle_forward_debug(w, rows=None):
    """The oracle's O and its per-row diagnostics (8-bit codes "pu8" [rows, N], ...)."""
    q, k, v = oracle_qkv(w)
    return oracle.get().attention_fwd(q, k, v, oracle_bias(w), block_c=128, rows=rows, debug=True)


def sample_rows(N: int, n: int = 48, seed: int = 0) -> np.ndarray:
    """First and last rows (the ragged tail) plus random rows in between, sorted."""
    rng = np.random.default_rng(seed)
    fixed = {0, 1, N - 1, N - 2, N // 2}
    extra = rng.choice(N, size=min(N, n), replace=False)
    rows = sorted({r for r in list(fixed) + list(extra) if 0 <= r < N})
    return np.array(rows, dtype=np.int64)


def o_errors(got: np.ndarray, want: np.ndarray):
    diff = np.abs(got.astype(np.float64) - want.astype(np.float64))
    return float(diff.max()) if diff.size else 0.0, float(diff.mean()) if diff.size else 0.0


def assert_o_close(got: np.ndarray, want: np.ndarray, what: str = ""):
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    mx, mean = o_errors(got, want)
    if what:
        record_parity(what, mx, mean)
    assert mx <= O_MAX_ABS and mean <= O_MEAN_ABS, f"{what}: max-abs {mx:.3g}, mean-abs {mean:.3g}"
    return mx, mean
