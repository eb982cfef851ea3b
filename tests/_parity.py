"""Shared comparison helpers for the GPU parity tests (test infrastructure)."""
import numpy as np
import torch

# Tolerances for bf16 outputs against the fp64 oracle: max-abs 1e-2 and
# mean-abs 1e-3 on the attention output, 1e-3 on the natural-log LSE.
OUT_MAX = 1e-2
OUT_MEAN = 1e-3
LSE_MAX = 1e-3


def assert_out_close(got, ref, what="out"):
    """max-abs 1e-2 / mean-abs 1e-3 against the fp64 oracle.  The max bound is
    applied beyond the output's own bf16 quantization: rounding a value r to
    bf16 alone moves it by up to 2^-9 * 2^ceil(log2|r|) <= 2^-8 |r|, which is
    already 0.0156 for |r| in [4, 8), so the per-element bound is
    1e-2 + 2^-8 |r|."""
    g = got.detach().float().cpu().numpy().astype(np.float64).reshape(ref.shape)
    err = np.abs(g - ref)
    assert np.all(np.isfinite(g)), f"{what}: non-finite output"
    excess = err - 2.0 ** -8 * np.abs(ref)
    mx, mean = float(excess.max(initial=0.0)), float(err.mean()) if err.size else 0.0
    assert mx <= OUT_MAX, f"{what}: max-abs beyond bf16 rounding {mx:.3e} > {OUT_MAX}"
    assert mean <= OUT_MEAN, f"{what}: mean-abs {mean:.3e} > {OUT_MEAN}"
    return mx, mean


def assert_lse_close(got, ref, what="lse"):
    g = got.detach().float().cpu().numpy().astype(np.float64).reshape(ref.shape)
    both_inf = np.isneginf(g) & np.isneginf(ref)
    assert np.array_equal(np.isneginf(g), np.isneginf(ref)), f"{what}: -inf pattern differs"
    err = np.abs(np.where(both_inf, 0.0, g - np.where(both_inf, 0.0, ref)))
    mx = float(err.max(initial=0.0))
    assert mx <= LSE_MAX, f"{what}: max-abs {mx:.3e} > {LSE_MAX}"
    return mx


def sample_rows(n_all, n_sample, seed=0, edge=64):
    """Sorted, de-duplicated sample: the first and last `edge` rows plus a
    seeded uniform sample."""
    rng = np.random.default_rng(seed)
    rows = set(range(min(edge, n_all))) | set(range(max(0, n_all - edge), n_all))
    rows |= set(rng.choice(n_all, size=min(n_sample, n_all), replace=False).tolist())
    return np.array(sorted(rows), dtype=np.int64)


def to_dev(d, dev="cuda"):
    return {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in d.items()}
