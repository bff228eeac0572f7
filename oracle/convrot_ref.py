"""CPU oracle for the ConvRot W8A8 / W4A8 linear layer.

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU
baseline / reference arm of ``bench.py`` may import this module.  The product
(the CUDA library and its Python binding) never imports, calls or links it,
and this module imports nothing from the product.

Everything is plain numpy in float64, written from the model cards' prose:

* "MOSS-Image Qwen3.5-9B text encoder, INT8 (W8A8, ConvRot)"
  - file table, "Quantized" row: every weight is rotated per 256-column group
    by a Hadamard matrix and stored as int8 with one fp32 ``weight_scale`` per
    output row;
  - file table, "Matmul" row: the input is rotated by the same Hadamard and
    rounded to int8 per token; the matmul is W8A8;
  - file table, "Changed" row and "How it was made": the decoder RMSNorm
    weights (fp32) carry SmoothQuant scales folded as (1 + w) / s - 1, with
    alpha = 0.5.
* "Qwen3.5 INT8 ConvRot Text Encoders for ComfyUI", "Why ConvRot" and
  "Quantization Recipe": group-wise Hadamard rotation with group size 256,
  row-wise scaling, plain rounding (``--simple``).
* "Qwen3-VL-8B-Heretic-1.3.0 - INT8 ConvRot (ComfyUI)", "Quantization
  metadata": convrot, convrot_groupsize 256, per_row true.
* "Qwen3-VL 8B - INT8 ConvRot", "Layer and group selection": an input width
  that the group size does not divide falls back to plain row-wise INT8
  (``group = 0`` here).
* "Qwen3-VL-8B-Heretic-1.3.0 - INT8 ConvRot (ComfyUI)", "Precision layout":
  the quantised projections include mlp.gate_proj, mlp.up_proj and
  mlp.down_proj; the MOSS-Image card's "How it was made" folds down_proj's
  SmoothQuant scales into up_proj's rows.  The pages do not name the MLP's
  activation; the Qwen-family reading down(SiLU(gate(x)) * up(x)) is taken.
* "MossInt4", "Format": the convrot_w4a4 layout - 256-wide Hadamard, signed
  4-bit codes two per byte, one F32 scale per row chosen by a per-row clip
  search; activations stay 8-bit.

Readings of points the pages leave open (each is also listed in the design
notes): Sylvester natural-order Hadamard normalised by 1/sqrt(256), no random
signs; symmetric absmax scaling with codes clamped to +-qmax (127, or 7 for
int4) and round-half-even; a zero row gets scale 0 and all-zero codes; the
RMSNorm is x * (mean(x^2) + eps)^-1/2 * (1 + w) with no intermediate rounding;
the int4 clip grid is clip_lo + (clip_hi - clip_lo) * i / (steps - 1), error
is the row's sum of squared reconstruction errors, ties keep the smaller clip;
the low nibble of byte j holds code 2j; gate and up rows of the fused MLP
linear alternate in blocks of 16 rows, g and u are not rounded before
SiLU(g) * u, and only h is rounded to bf16; the down_proj fold into up_proj's
rows is applied to their row scales (exact for per-row quantisation).

Parity status: every function below is pinned by ``tests/test_oracle.py``
(closed forms, invariants, brute force on tiny inputs, library routines for
special cases, the pages' printed facts); none is "parity unpinned".  What is
NOT pinned is agreement with real ComfyUI checkpoint files (their Hadamard
ordering and sign convention), because no such file is available.
"""
from __future__ import annotations

import numpy as np

GROUP = 256          # "convrot_groupsize": 256
QMAX_INT8 = 127      # symmetric int8 codes, -128 never produced
QMAX_INT4 = 7        # symmetric signed 4-bit codes


# --------------------------------------------------------------------------
# Hadamard rotation
# --------------------------------------------------------------------------
def hadamard(n: int = GROUP) -> np.ndarray:
    """Normalised Sylvester Hadamard matrix H_n / sqrt(n) (float64, n = 2^k).

    Built by repeated Kronecker products of [[1, 1], [1, -1]]; entry (i, j) is
    (-1)^popcount(i & j) / sqrt(n).  The matrix is symmetric and orthogonal,
    so rotating by H or by H^T is the same operation.
    """
    if n < 1 or n & (n - 1):
        raise ValueError("Hadamard size must be a power of two")
    base = np.array([[1.0, 1.0], [1.0, -1.0]])
    h = np.ones((1, 1))
    while h.shape[0] < n:
        h = np.kron(base, h)
    return h / np.sqrt(n)


def rotate_groups(a, group: int = GROUP) -> np.ndarray:
    """a @ blockdiag(H, ..., H) along the last axis (the input dimension K).

    Column block g = [g*group, (g+1)*group) is multiplied by H.  group = 0 is
    the plain row-wise fallback: no rotation.
    """
    a = np.asarray(a, dtype=np.float64)
    if group == 0:
        return a.copy()
    K = a.shape[-1]
    if K % group:
        raise ValueError(f"K={K} is not a multiple of the group size {group}")
    h = hadamard(group)
    lead = a.shape[:-1]
    blocks = a.reshape(*lead, K // group, group)
    return (blocks @ h).reshape(*lead, K)


# --------------------------------------------------------------------------
# symmetric absmax quantisation (per row)
# --------------------------------------------------------------------------
def absmax_quantize(v, qmax: int):
    """Per-row symmetric quantisation.

    s = max_k |v[k]| / qmax; q = clamp(rint(v / s), -qmax, qmax) with
    round-half-even; a row with max 0 gets s = 0 and q = 0.
    Returns (q as int64, s as float64).
    """
    v = np.asarray(v, dtype=np.float64)
    amax = np.max(np.abs(v), axis=-1)
    s = amax / qmax
    safe = np.where(s > 0, s, 1.0)
    q = np.rint(v / safe[..., None])
    q = np.where((s > 0)[..., None], q, 0.0)
    q = np.clip(q, -qmax, qmax)
    return q.astype(np.int64), s


# --------------------------------------------------------------------------
# weights (offline)
# --------------------------------------------------------------------------
def quantize_weight(W, group: int = GROUP, col_scale=None):
    """ConvRot int8 weight: optional column scale, group rotation, per-row int8.

    W [N, K] -> (Wq int8 [N, K], s_row float32 [N], W' float64 [N, K]).
    The per-row scale is stored as fp32, the precision the cards give for
    ``weight_scale`` (file table of the MOSS-Image card; F32 scale tensors in
    the Heretic card's "Verification").  The codes are decided in float64.
    """
    Wd = np.asarray(W, dtype=np.float64)
    if col_scale is not None:
        Wd = Wd * np.asarray(col_scale, dtype=np.float64)[None, :]
    Wr = rotate_groups(Wd, group)
    q, s = absmax_quantize(Wr, QMAX_INT8)
    return q.astype(np.int8), s.astype(np.float32), Wr


def clip_grid(clip_lo: float, clip_hi: float, steps: int) -> np.ndarray:
    """Clip candidates clip_lo + (clip_hi - clip_lo) * i / (steps - 1)."""
    if steps == 1:
        return np.array([float(clip_hi)])
    i = np.arange(steps, dtype=np.float64)
    return float(clip_lo) + (float(clip_hi) - float(clip_lo)) * i / (steps - 1)


def quantize_weight_w4(W, group: int = GROUP, col_scale=None, clip_lo: float = 0.80,
                       clip_hi: float = 1.00, clip_steps: int = 21):
    """convrot_w4a4 weight layout ("MossInt4", "Format").

    Rotate, then per row try every clip c of the grid: s = c * max|W'| / 7,
    q = clamp(rint(W' / s), -7, 7), err = sum (W' - s q)^2; keep the smallest
    error (the first, i.e. smallest c, on ties).
    Returns dict with codes int8 [N,K], s_row float32 [N], s64 float64 [N],
    clip float64 [N], err float64 [N], packed uint8 [N, K/2], rotated W'.
    """
    Wd = np.asarray(W, dtype=np.float64)
    if col_scale is not None:
        Wd = Wd * np.asarray(col_scale, dtype=np.float64)[None, :]
    Wr = rotate_groups(Wd, group)
    amax = np.max(np.abs(Wr), axis=1)
    N = Wr.shape[0]
    best_err = np.full(N, np.inf)
    best_s = np.zeros(N)
    best_c = np.zeros(N)
    best_q = np.zeros(Wr.shape, dtype=np.int64)
    for c in clip_grid(clip_lo, clip_hi, clip_steps):
        s = c * amax / QMAX_INT4
        safe = np.where(s > 0, s, 1.0)
        q = np.clip(np.rint(Wr / safe[:, None]), -QMAX_INT4, QMAX_INT4)
        q = np.where((s > 0)[:, None], q, 0.0)
        err = np.sum((Wr - s[:, None] * q) ** 2, axis=1)
        better = err < best_err
        best_err = np.where(better, err, best_err)
        best_s = np.where(better, s, best_s)
        best_c = np.where(better, c, best_c)
        best_q[better] = q[better].astype(np.int64)
    return {
        "codes": best_q.astype(np.int8),
        "s_row": best_s.astype(np.float32),
        "s64": best_s,
        "clip": best_c,
        "err": best_err,
        "packed": pack_int4(best_q),
        "rotated": Wr,
    }


def pack_int4(codes) -> np.ndarray:
    """Two signed 4-bit codes per byte: code 2j in bits 0-3, code 2j+1 in bits 4-7."""
    c = np.asarray(codes, dtype=np.int64)
    if c.shape[-1] % 2:
        raise ValueError("K must be even to pack two codes per byte")
    if c.min(initial=0) < -8 or c.max(initial=0) > 7:
        raise ValueError("codes out of the signed 4-bit range")
    lo = c[..., 0::2] & 0xF
    hi = c[..., 1::2] & 0xF
    return (lo | (hi << 4)).astype(np.uint8)


def unpack_int4(packed) -> np.ndarray:
    """Inverse of pack_int4: uint8 [.., K/2] -> int8 codes [.., K]."""
    p = np.asarray(packed, dtype=np.int64)
    lo = p & 0xF
    hi = (p >> 4) & 0xF
    lo = np.where(lo >= 8, lo - 16, lo)
    hi = np.where(hi >= 8, hi - 16, hi)
    out = np.empty(p.shape[:-1] + (2 * p.shape[-1],), dtype=np.int64)
    out[..., 0::2] = lo
    out[..., 1::2] = hi
    return out.astype(np.int8)


# --------------------------------------------------------------------------
# activations (online)
# --------------------------------------------------------------------------
def rmsnorm(x, norm_w, eps: float):
    """x * (mean_k x^2 + eps)^(-1/2) * (1 + w), float64, no intermediate rounding.

    The (1 + w) form is the one the MOSS-Image card's "How it was made" folds
    the SmoothQuant scale into.  eps is taken at the fp32 value the library
    receives.
    """
    x = np.asarray(x, dtype=np.float64)
    e = float(np.float32(eps))
    ms = np.mean(x * x, axis=-1) + e
    # an all-zero row with eps = 0 stays zero (scale 0, codes 0) instead of 0/0
    r = np.where(ms > 0, 1.0 / np.sqrt(np.where(ms > 0, ms, 1.0)), 0.0)
    return x * r[..., None] * (1.0 + np.asarray(norm_w, dtype=np.float64))[None, :]


def rotate_quant_act(x, group: int = GROUP, norm_w=None, eps: float = 1e-6):
    """Online activation path: [RMSNorm] -> group Hadamard -> per-token int8.

    x [M, K] -> (Xq int8 [M, K], s_tok float64 [M], v float64 [M, K]) where v
    is the rotated (and normalised) activation the codes are taken from.
    """
    u = np.asarray(x, dtype=np.float64)
    if norm_w is not None:
        u = rmsnorm(u, norm_w, eps)
    v = rotate_groups(u, group)
    q, s = absmax_quantize(v, QMAX_INT8)
    return q.astype(np.int8), s, v


# --------------------------------------------------------------------------
# integer matmul and dequantisation
# --------------------------------------------------------------------------
def int_matmul(A, B) -> np.ndarray:
    """acc[m, n] = sum_k A[m, k] * B[n, k], exact, as int64.

    Evaluated as a float64 product of integer-valued matrices: every partial
    sum is an integer below 2^53 in magnitude, so the result is exact in any
    summation order (checked by the bound below).
    """
    A = np.asarray(A)
    B = np.asarray(B)
    K = A.shape[1]
    bound = int(np.abs(A).max(initial=0)) * int(np.abs(B).max(initial=0)) * K
    if bound >= 2 ** 53:
        raise ValueError("integer matmul would not be exact in float64")
    return (A.astype(np.float64) @ B.astype(np.float64).T).astype(np.int64)


def dequant(acc, s_tok, s_row) -> np.ndarray:
    """y = acc * s_tok[m] * s_row[n] in float64."""
    return (np.asarray(acc, dtype=np.float64)
            * np.asarray(s_tok, dtype=np.float64)[:, None]
            * np.asarray(s_row, dtype=np.float64)[None, :])


def to_bf16(y) -> np.ndarray:
    """Round float64 values to the nearest bfloat16 (ties to even), as float64.

    bfloat16 keeps 8 significant bits: with y = m * 2^e, 0.5 <= |m| < 1, the
    result is rint(m * 2^8) * 2^(e - 8).  Exponents below the normal range
    are clamped so that subnormals round on the 2^-133 grid.
    """
    y = np.asarray(y, dtype=np.float64)
    _, e = np.frexp(y)
    e = np.maximum(e, -125)
    q = np.rint(np.ldexp(y, 8 - e))
    return np.ldexp(q, e - 8)


def int8_linear(Xq, s_tok, Wq, s_row):
    """W8A8 linear: bf16(acc * s_tok * s_row). Returns (y_bf16, y64, acc)."""
    acc = int_matmul(Xq, Wq)
    y = dequant(acc, s_tok, s_row)
    return to_bf16(y), y, acc


def w4a8_linear(Xq, s_tok, packed, s_row):
    """W4A8 linear on packed int4 weights; same accumulation and dequant."""
    return int8_linear(Xq, s_tok, unpack_int4(packed), s_row)


def linear_forward(x, Wq, s_row, group: int = GROUP, norm_w=None, eps: float = 1e-6):
    """Whole online path: rotate-quantise the activation, then the W8A8 linear."""
    Xq, s_tok, _ = rotate_quant_act(x, group, norm_w, eps)
    yb, y, acc = int8_linear(Xq, s_tok, Wq, s_row)
    return yb, {"Xq": Xq, "s_tok": s_tok, "acc": acc, "y64": y}


# --------------------------------------------------------------------------
# SmoothQuant calibration used to prepare the synthetic norm-carrying layer
# --------------------------------------------------------------------------
def smoothquant_scales_of(a, W, alpha: float = 0.5, s_min: float = 1e-5, s_max: float = 1e5):
    """Per input channel s_c = max_m|a[m,c]|^alpha / max_n|W[n,c]|^(1-alpha).

    ``a`` [M, K] is the activation exactly as it reaches the linear (MOSS-Image
    card, "How it was made": SmoothQuant, alpha 0.5, per input channel).  s is
    clamped to [s_min, s_max]; a channel whose activation or weight column is
    all zero keeps s = 1.
    """
    ax = np.max(np.abs(np.asarray(a, dtype=np.float64)), axis=0)
    aw = np.max(np.abs(np.asarray(W, dtype=np.float64)), axis=0)
    ok = (ax > 0) & (aw > 0)
    s = np.where(ok, np.power(np.where(ok, ax, 1.0), alpha)
                 / np.power(np.where(ok, aw, 1.0), 1.0 - alpha), 1.0)
    return np.clip(s, s_min, s_max)


def smoothquant_scales(x, norm_w, eps: float, W, alpha: float = 0.5,
                       s_min: float = 1e-5, s_max: float = 1e5):
    """Per input channel s_c = max_m|a[m,c]|^alpha / max_n|W[n,c]|^(1-alpha).

    a = RMSNorm(x) * (1 + w) is the activation that reaches the linear; the
    scale moves activation outliers into the weight (MOSS-Image card, "How it
    was made", alpha 0.5).  s is clamped to [s_min, s_max]; a channel whose
    activation or weight column is all zero keeps s = 1.  Returns
    (s, w_folded) with w_folded = (1 + w) / s - 1, the stored norm weight;
    the weight is then used as W * diag(s).
    """
    s = smoothquant_scales_of(rmsnorm(x, norm_w, eps), W, alpha, s_min, s_max)
    w_folded = (1.0 + np.asarray(norm_w, dtype=np.float64)) / s - 1.0
    return s, w_folded


# --------------------------------------------------------------------------
# weight-only path: rotated activations kept in bf16, int8 weight codes
# --------------------------------------------------------------------------
def rotate_act(x, group: int = GROUP, norm_w=None, eps: float = 1e-6) -> np.ndarray:
    """[RMSNorm] then the group rotation, without quantisation (float64).

    The MOSS-Image card's "Matmul" row: the weight can also be dequantised for a
    bf16 matmul.  A ConvRot weight is stored rotated (W' = W R), and
    x W^T = (x R) W'^T, so the activation is rotated instead of the weight
    being rotated back.
    """
    u = np.asarray(x, dtype=np.float64)
    if norm_w is not None:
        u = rmsnorm(u, norm_w, eps)
    return rotate_groups(u, group)


def weight_only_linear(Xr, Wq, s_row):
    """y[m,n] = s_row[n] * sum_k Xr[m,k] Wq[n,k] (float64), and its bf16 rounding.

    Xr is the rotated activation as the GEMM receives it (bf16 values);
    returns (y_bf16, y64)."""
    y = (np.asarray(Xr, dtype=np.float64) @ np.asarray(Wq, dtype=np.float64).T
         * np.asarray(s_row, dtype=np.float64)[None, :])
    return to_bf16(y), y


# --------------------------------------------------------------------------
# MLP boundary: gate/up linear with SiLU(gate) * up, and the down_proj fold
# --------------------------------------------------------------------------
SWIGLU_BLOCK = 16  # gate and up rows alternate in blocks of this many rows


def silu(z) -> np.ndarray:
    """SiLU(z) = z * sigmoid(z) = z / (1 + exp(-z)), float64.

    Evaluated as z * e / (1 + e) with e = exp(z) for z < 0 so that exp never
    overflows; both forms are the same function.
    """
    z = np.asarray(z, dtype=np.float64)
    pos = z >= 0
    ez = np.exp(np.where(pos, -z, z))          # in (0, 1]
    sig = np.where(pos, 1.0 / (1.0 + ez), ez / (1.0 + ez))
    return z * sig


def interleave_gate_up(Wg, Wu, block: int = SWIGLU_BLOCK) -> np.ndarray:
    """Rows of gate and up in alternating blocks: [g0..g15, u0..u15, g16..].

    Wg, Wu [I, ...] -> [2I, ...]; row r of the result is gate row
    block*(r // (2 block)) + r % (2 block) when r % (2 block) < block, else
    the up row with the same index.  I % block == 0.  One tile row of 2*block
    accumulators then holds matching gate and up columns, which lets the
    GEMM epilogue form SiLU(gate) * up without another pass.
    """
    Wg = np.asarray(Wg)
    Wu = np.asarray(Wu)
    if Wg.shape != Wu.shape or Wg.shape[0] % block:
        raise ValueError("gate and up must have the same shape with rows a multiple of the block")
    I = Wg.shape[0]
    out = np.empty((2 * I,) + Wg.shape[1:], dtype=np.result_type(Wg, Wu))
    gv = Wg.reshape((I // block, block) + Wg.shape[1:])
    uv = Wu.reshape((I // block, block) + Wu.shape[1:])
    ov = out.reshape((I // block, 2, block) + Wg.shape[1:])
    ov[:, 0] = gv
    ov[:, 1] = uv
    return out


def swiglu_linear(Xq, s_tok, Wq_gu, s_row_gu, block: int = SWIGLU_BLOCK):
    """h = SiLU(g) * u from one W8A8 GEMM over interleaved gate/up weights.

    g and u are the dequantised products acc * s_tok * s_row (float64, no
    rounding before the activation); h [M, I] is rounded once to bf16.  This
    is the down_proj input of a Qwen MLP block, down(SiLU(gate(x)) * up(x)).
    Returns (h_bf16, h64, y64) with y64 the interleaved [M, 2I] products.
    """
    acc = int_matmul(Xq, Wq_gu)
    y = dequant(acc, s_tok, s_row_gu)
    M, N2 = y.shape
    yv = y.reshape(M, N2 // (2 * block), 2, block)
    g = yv[:, :, 0, :].reshape(M, N2 // 2)
    u = yv[:, :, 1, :].reshape(M, N2 // 2)
    h = silu(g) * u
    return to_bf16(h), h, y


def fold_smooth_into_rows(s_row, smooth) -> np.ndarray:
    """Fold a per-channel scale 1/s into the rows of a row-quantised weight.

    down_proj's SmoothQuant scale goes "into up_proj's rows" (MOSS-Image card,
    "How it was made").  Each row of a ConvRot weight is rotated and quantised
    on its own with an absmax scale, so dividing row c by s_c leaves its codes
    unchanged and divides its scale: the fold is s_row[c] / s_c.
    """
    return np.asarray(s_row, dtype=np.float64) / np.asarray(smooth, dtype=np.float64)
