"""Shared helpers of the GPU parity tests: tolerances and row sampling.

Tolerances
  fp32 path: max_i |o - o*| / max |o*| <= 1e-5 (norm-wise relative).
  bf16 path: max |o - o*| <= 2e-2 and mean |o - o*| <= 2e-3 over all checked
  elements, plus a tighter check derived from the arithmetic: each bf16
  operand rounding (P, phi(Q), S for the linear term, phi(K) inside S) has
  relative error <= 2^-8 and the roundings are independent across the
  thousands of keys a row sums over, so the error of a row is a random sum
  whose rms is about 2^-8 * rms(o*). The test allows rms(o - o*) <=
  4e-2 * rms(o*), ten times that estimate.
"""
import numpy as np
import torch

F32_REL = 1e-5
BF16_MAX_ABS = 2e-2
BF16_MEAN_ABS = 2e-3
BF16_REL_RMS = 4e-2


def errors(o, ref):
    o = np.asarray(o, np.float64)
    ref = np.asarray(ref, np.float64)
    d = np.abs(o - ref)
    return {
        "max_abs": float(d.max()),
        "mean_abs": float(d.mean()),
        "rel_max": float(d.max() / max(np.abs(ref).max(), 1e-300)),
        "rel_rms": float(np.sqrt((d ** 2).mean()) / max(np.sqrt((ref ** 2).mean()), 1e-300)),
    }


def assert_f32(o, ref, what=""):
    e = errors(o, ref)
    assert np.all(np.isfinite(o)), what
    assert e["rel_max"] <= F32_REL, (what, e)
    return e


def assert_bf16(o, ref, what=""):
    e = errors(o, ref)
    assert np.all(np.isfinite(o)), what
    assert e["max_abs"] <= BF16_MAX_ABS, (what, e)
    assert e["mean_abs"] <= BF16_MEAN_ABS, (what, e)
    assert e["rel_rms"] <= BF16_REL_RMS, (what, e)
    return e


def assert_bf16_peaked(o, ref, v, what=""):
    """bf16 check for inputs whose softmax is nearly one-hot (large logits).

    There a row's output is close to a single value row, so |o*| reaches max |v| and the
    fixed 2e-2 bound of assert_bf16 stops following from the arithmetic. The bound used
    instead: rounding o to bf16 costs <= 2^-8 |o*|; rounding each p to bf16 perturbs the
    numerator by <= 2^-8 sum_j p_j |v_j| <= 2^-8 l max|v| while l is summed from the
    unrounded p, so it costs <= 2^-8 max|v| (max over the head). Together
    |o - o*| <= 2^-8 (|o*| + max|v|), plus the mean-abs and rms checks of assert_bf16.
    """
    o = np.asarray(o, np.float64)
    ref = np.asarray(ref, np.float64)
    e = errors(o, ref)
    assert np.all(np.isfinite(o)), what
    vmax = np.abs(np.asarray(v, np.float64)).max(axis=(2, 3), keepdims=True)
    bound = 2.0 ** -8 * (np.abs(ref) + vmax) + 1e-6
    worst = float((np.abs(o - ref) / bound).max())
    assert worst <= 1.0, (what, e, worst)
    assert e["mean_abs"] <= BF16_MEAN_ABS, (what, e)
    assert e["rel_rms"] <= BF16_REL_RMS, (what, e)
    return e


def assert_parity(dtype, o, ref, what=""):
    return assert_f32(o, ref, what) if dtype == "f32" else assert_bf16(o, ref, what)


def sample_rows(n_rows, tile_starts, per_tile=3, seed=0, extra=()):
    """Rows covering the first/last row of given tiles plus random rows."""
    rng = np.random.default_rng(seed)
    rows = set(int(r) for r in extra)
    for t0, t1 in tile_starts:
        rows.update([t0, t1 - 1])
        rows.update(int(x) for x in rng.integers(t0, t1, size=per_tile))
    return np.array(sorted(r for r in rows if 0 <= r < n_rows), dtype=np.int64)


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu").to(torch.float64).numpy()
