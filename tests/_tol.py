"""Tolerances of the CUDA path against the float64 oracle, derived from the
fp32 arithmetic the kernels perform.

The kernels take every rounding decision in fp32 while the oracle takes it in
float64.  A code can therefore differ only where the oracle's value lies
within the fp32 error of a rounding tie; these helpers bound that error.

Error model (u = 2^-24, unit roundoff of fp32):
* inputs: bf16 values are exact in fp32; a per-column multiplier (RMSNorm
  weight 1 + w, or a column scale) adds at most 2u relative per element;
* FWHT: 8 butterfly stages, each stage's rounding error is at most u times the
  2-norm of that stage's output, and later stages scale errors by sqrt(2) per
  stage like the signal, so the error of a group's transform has 2-norm at
  most 8u * ||v_g||_2 (plus 2u * ||v_g||_2 from the inputs);
* per-row absmax: off by at most E = max_g 10u ||v_g||_2;
* codes: z = v * fp32(127 / absmax), two more roundings.
A factor of 1.5 covers second-order terms.
"""
import numpy as np

U = 2.0 ** -24


def row_error(v, group, pre, extra_rel=0.0):
    """E / absmax per row (0 for all-zero rows), for the rotated values v.

    extra_rel is an additional relative perturbation of the inputs, e.g. when
    the two sides derived a per-column multiplier independently."""
    v = np.asarray(v, dtype=np.float64)
    amax = np.max(np.abs(v), axis=1)
    in_rel = (2.0 * U if pre else 0.0) + extra_rel
    if group:
        M, K = v.shape
        gn = np.sqrt(np.sum(v.reshape(M, K // group, group) ** 2, axis=2)).max(axis=1)
        E = (8.0 * U + in_rel) * gn
    else:
        E = in_rel * amax
    with np.errstate(divide="ignore", invalid="ignore"):
        r = np.where(amax > 0, E / np.where(amax > 0, amax, 1.0), 0.0)
    return r, amax


def int8_code_window(ratio):
    """Half-width of the window around a tie in which an int8 code may flip."""
    return 1.5 * 127.0 * (2.0 * ratio + 2.0 * U)


def scale_rel_tol(ratio, norm):
    """Relative tolerance of the fp32 per-row scale against float64."""
    return 1.5 * (ratio + (5.0 if norm else 1.0) * U) + 2.0 * U


def check_codes(q_gpu, q_ref, z, window, name="codes"):
    """|q_gpu - q_ref| <= 1, and only where |frac(|z|) - 1/2| <= window (per row).

    Returns the number of differing codes.
    """
    q_gpu = np.asarray(q_gpu, dtype=np.int64)
    q_ref = np.asarray(q_ref, dtype=np.int64)
    diff = q_gpu - q_ref
    assert np.abs(diff).max(initial=0) <= 1, f"{name}: a code differs by more than 1"
    az = np.abs(z)
    dist = np.abs(az - np.floor(az) - 0.5)
    w = np.broadcast_to(np.asarray(window, dtype=np.float64)[:, None], dist.shape)
    bad = (diff != 0) & (dist > w)
    if bad.any():
        i, j = np.argwhere(bad)[0]
        raise AssertionError(f"{name}: code differs away from a tie at ({i},{j}): "
                             f"z={z[i, j]!r} gpu={q_gpu[i, j]} ref={q_ref[i, j]} "
                             f"dist={dist[i, j]:.3e} window={w[i, j]:.3e}")
    return int((diff != 0).sum())


def bf16_ulp(y):
    """Spacing of bfloat16 numbers at |y| (2^(e-7) for 2^e <= |y| < 2^(e+1))."""
    y = np.abs(np.asarray(y, dtype=np.float64))
    _, e = np.frexp(np.where(y > 0, y, 1.0))
    e = np.maximum(e - 1, -126)
    return np.ldexp(1.0, e - 7)


def output_tol(y_ref):
    """Output tolerance: |y - y_ref| <= 2^-7 |y_ref| + 1e-3 max_n |y_ref[m, :]|."""
    y_ref = np.asarray(y_ref, dtype=np.float64)
    return 2.0 ** -7 * np.abs(y_ref) + 1e-3 * np.max(np.abs(y_ref), axis=1, keepdims=True)


def check_w4_clip(wr, s_gpu, amax, best_err, ratio, grid):
    """The GPU's int4 clip choice for one row, checked against the float64
    clip search ("MossInt4", "Format": per-row clip search over a grid of
    clip factors, minimum row error).

    The GPU's scale must sit on the clip grid (within its fp32 error), and the
    float64 row error at that clip must be within the fp32 evaluation error of
    the float64 optimum `best_err`: the GPU evaluates every candidate in fp32,
    so two candidates closer than that bound are both acceptable choices.
    Returns (s64, q): the float64 scale of the chosen grid point and the
    oracle's codes at that scale, which the caller compares code by code.
    """
    wr = np.asarray(wr, dtype=np.float64)
    c_g = s_gpu * 7.0 / amax
    i_g = int(np.argmin(np.abs(grid - c_g)))
    assert abs(c_g - grid[i_g]) <= 1.5 * (ratio + 6 * U) * grid[i_g], "s_row off the clip grid"
    s64 = grid[i_g] * amax / 7.0
    q = np.clip(np.rint(wr / s64), -7, 7)
    err_g = np.sum((wr - s64 * q) ** 2)
    v2 = np.linalg.norm(wr)
    # error of one fp32 candidate evaluation: the rotated row (10u ||v||), the
    # reconstruction s q (its scale's relative error) and the sum of squares
    dd = 10 * U * v2 + np.linalg.norm(q) * s64 * (ratio + 3 * U) + 2 * U * v2
    tol_sse = 2 * (2 * np.sqrt(best_err + err_g) * dd + 2 * dd * dd + 48 * U * err_g)
    # codes inside the tie window may round either way on the GPU
    win4 = int4_code_window(ratio)
    z = wr / s64
    near = np.abs(np.abs(z) - np.floor(np.abs(z)) - 0.5) <= win4
    tol_sse += near.sum() * 2 * win4 * s64 * s64
    assert err_g <= best_err + tol_sse, f"clip {grid[i_g]}: row error {err_g} vs best {best_err}"
    return s64, q


def int4_code_window(ratio):
    """Half-width of the window around a tie in which an int4 code may flip."""
    return 1.5 * 8.75 * (2.0 * ratio + 4.0 * U)
