"""Shared helpers of the GPU parity tests (comparison metrics and tolerances).

Tolerances for bf16 outputs against the fp64 oracle: max-abs <= 2e-2 and
relative L2 <= 5e-3; e4m3 cache bytes and scales bit-exact; attention over an
e4m3 cache: relative L2 <= 2e-2 against the oracle reading the same bytes."""
import numpy as np
import torch

MAX_ABS = 2e-2
REL_L2 = 5e-3
REL_L2_FP8 = 2e-2


def to_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def errors(got: np.ndarray, want: np.ndarray):
    diff = got - want
    max_abs = float(np.abs(diff).max()) if diff.size else 0.0
    den = float(np.linalg.norm(want))
    rel = float(np.linalg.norm(diff) / den) if den > 0 else float(np.linalg.norm(diff))
    return max_abs, rel


def assert_parity(got, want, rel_l2=REL_L2, max_abs=MAX_ABS, what=""):
    got = to_f64(got) if isinstance(got, torch.Tensor) else got
    assert got.shape == want.shape, (got.shape, want.shape)
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    ma, rl = errors(got, want)
    assert ma <= max_abs and rl <= rel_l2, f"{what}: max_abs={ma:.3e} rel_l2={rl:.3e}"
    return ma, rl


def sample_rows(n_rows: int, k: int, seed: int, boundaries=()):
    """k random rows plus every boundary b-1, b, b+1 inside [0, n_rows)."""
    rng = np.random.default_rng(seed)
    rows = set(rng.choice(n_rows, size=min(k, n_rows), replace=False).tolist())
    for b in boundaries:
        for r in (b - 1, b, b + 1):
            if 0 <= r < n_rows:
                rows.add(r)
    rows.update({0, n_rows - 1})
    return np.array(sorted(rows), dtype=np.int64)
