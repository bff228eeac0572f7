"""Pins for the CPU oracle: checks against the pages' printed facts, closed
forms, invariants, brute force on tiny inputs and library routines.

None of these tests retypes an oracle formula to compare it with itself; each
check is chosen so that a plausible slip in the oracle (wrong normalisation or
ordering of H, rotation on the wrong axis or across group borders, a dropped
(1 + w), wrong rounding mode, a transposed operand, a wrong int4 nibble order
or clip tie-break) makes at least one of them fail.
"""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

from oracle import convrot_ref as ref

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _popsign(i, j):
    return -1.0 if bin(i & j).count("1") % 2 else 1.0


# ---------------------------------------------------------------- Hadamard
def test_hadamard_orthogonal_bit_exact():
    h = ref.hadamard(256)
    # entries are +-1/16, every product is +-1/256 and every partial sum is a
    # multiple of 1/256 below 1: float64 computes H H^T exactly
    assert np.array_equal(h @ h.T, np.eye(256))
    assert np.array_equal(h, h.T)


def test_hadamard_entries_popcount():
    h = ref.hadamard(256) * 16.0
    for i in range(256):
        for j in range(256):
            assert h[i, j] == _popsign(i, j)


def test_hadamard_small_sylvester_textbook():
    assert np.array_equal(ref.hadamard(2) * math.sqrt(2), [[1, 1], [1, -1]])
    h4 = [[1, 1, 1, 1], [1, -1, 1, -1], [1, 1, -1, -1], [1, -1, -1, 1]]
    assert np.allclose(ref.hadamard(4) * 2, h4, rtol=0, atol=0)


def test_group_size_matches_card_metadata():
    meta = _golden("comfy_quant_metadata.json")["metadata"]
    assert meta["convrot"] is True
    assert ref.GROUP == meta["convrot_groupsize"] == 256
    assert meta["per_row"] is True


# ---------------------------------------------------------------- rotation
def test_rotation_preserves_products():
    rng = np.random.default_rng(0)
    x = rng.standard_normal((5, 768))
    W = rng.standard_normal((7, 768))
    lhs = ref.rotate_groups(x) @ ref.rotate_groups(W).T
    rhs = x @ W.T
    assert np.max(np.abs(lhs - rhs)) <= 1e-12 * np.max(np.abs(rhs)) * 10


def test_rotation_one_hot_stays_in_its_group():
    K = 768
    for g, j in [(0, 0), (1, 5), (2, 255), (1, 128)]:
        x = np.zeros((1, K))
        x[0, 256 * g + j] = 1.0
        v = ref.rotate_groups(x)[0]
        for gg in range(3):
            blk = v[256 * gg: 256 * gg + 256]
            if gg != g:
                assert not blk.any()
            else:
                expect = np.array([_popsign(i, j) / 16 for i in range(256)])
                assert np.array_equal(blk, expect)


def test_rotation_constant_group():
    x = np.zeros((1, 512))
    x[0, 256:] = 3.0
    v = ref.rotate_groups(x)[0]
    assert np.array_equal(v[:256], np.zeros(256))
    assert v[256] == 48.0 and not v[257:].any()


def test_rotation_brute_force_tiny():
    rng = np.random.default_rng(1)
    x = rng.integers(-4, 5, size=(1, 512)).astype(np.float64)
    got = ref.rotate_groups(x)[0]
    for g in range(2):
        for i in range(0, 256, 17):
            s = sum(x[0, 256 * g + j] * _popsign(i, j) for j in range(256)) / 16
            assert got[256 * g + i] == s


def test_hadamard_16_for_the_vision_group():
    # "Qwen3-VL 8B - INT8 ConvRot", "Layer and group selection": group size 16
    # for vision widths 1152 and 4304, which 256 does not divide but 16 does
    h = ref.hadamard(16)
    assert np.array_equal(h @ h.T, np.eye(16)) and np.array_equal(h, h.T)
    for i in range(16):
        for j in range(16):
            assert h[i, j] * 4.0 == _popsign(i, j)
    assert 1152 % 256 and 4304 % 256 and not 1152 % 16 and not 4304 % 16


def test_rotation_group16_brute_force():
    rng = np.random.default_rng(4)
    x = rng.integers(-4, 5, size=(2, 48)).astype(np.float64)
    got = ref.rotate_groups(x, 16)
    for r in range(2):
        for g in range(3):
            for i in range(16):
                s = sum(x[r, 16 * g + j] * _popsign(i, j) for j in range(16)) / 4
                assert got[r, 16 * g + i] == s
    # products survive the rotation as for 256-groups
    W = rng.standard_normal((5, 1152))
    xx = rng.standard_normal((3, 1152))
    np.testing.assert_allclose(ref.rotate_groups(xx, 16) @ ref.rotate_groups(W, 16).T, xx @ W.T,
                               rtol=1e-12, atol=1e-12)


def test_group_zero_is_plain_rowwise():
    rng = np.random.default_rng(2)
    x = rng.standard_normal((3, 48))
    assert np.array_equal(ref.rotate_groups(x, 0), x)
    with pytest.raises(ValueError):
        ref.rotate_groups(x, 256)


# ---------------------------------------------------------------- quantisation
def test_absmax_invariants():
    rng = np.random.default_rng(3)
    v = rng.standard_normal((64, 512)) * rng.uniform(0.01, 10, size=(64, 1))
    q, s = ref.absmax_quantize(v, 127)
    assert np.abs(q).max() <= 127
    am = np.argmax(np.abs(v), axis=1)
    assert np.array_equal(q[np.arange(64), am], 127 * np.sign(v[np.arange(64), am]))
    assert np.all(np.abs(v - s[:, None] * q) <= s[:, None] * (0.5 + 1e-12))


def test_absmax_zero_row_and_rne_ties():
    v = np.array([[0.0] * 8,
                  [127.0, 2.5, -2.5, 3.5, 0.5, -0.5, 1.5, -126.5]])
    q, s = ref.absmax_quantize(v, 127)
    assert s[0] == 0.0 and not q[0].any()
    assert s[1] == 1.0
    # python's round() is round-half-even
    assert list(q[1]) == [round(t) for t in v[1]] == [127, 2, -2, 4, 0, 0, 2, -126]


def test_absmax_matches_python_round_brute_force():
    rng = np.random.default_rng(4)
    v = rng.standard_normal((3, 40))
    q, s = ref.absmax_quantize(v, 127)
    for r in range(3):
        amax = max(abs(t) for t in v[r])
        for k in range(40):
            assert q[r, k] == max(-127, min(127, round(v[r, k] / (amax / 127))))


def test_weight_one_scale_per_output_row():
    census = _golden("tensor_census.json")
    assert census["int8_tensors"] == census["f32_scale_tensors"]
    assert census["blocks"] * len(census["projections_per_block"]) == census["int8_tensors"]
    rng = np.random.default_rng(5)
    W = rng.standard_normal((6, 512)) * 0.02
    Wq, s, _ = ref.quantize_weight(W)
    assert Wq.dtype == np.int8 and Wq.shape == W.shape
    assert s.dtype == np.float32 and s.shape == (6,)


def test_weight_quant_rotates_columns_not_rows():
    # a weight with one nonzero column j in group g: after rotation each row is
    # w[n] * row j of H in group g; every code is +-127
    W = np.zeros((3, 512))
    W[:, 256 + 9] = [1.0, -2.0, 0.5]
    Wq, s, _ = ref.quantize_weight(W)
    assert not Wq[:, :256].any()
    expect = np.array([127 * _popsign(i, 9) for i in range(256)])
    assert np.array_equal(Wq[0, 256:], expect)
    assert np.array_equal(Wq[1, 256:], -expect)
    assert np.allclose(s, np.float32(np.array([1.0, 2.0, 0.5]) / 16 / 127))


# ---------------------------------------------------------------- integer GEMM
def test_int_matmul_brute_force():
    rng = np.random.default_rng(6)
    for M, N, K in [(1, 1, 256), (3, 5, 256), (8, 8, 256), (2, 7, 32)]:
        A = rng.integers(-127, 128, size=(M, K))
        B = rng.integers(-127, 128, size=(N, K))
        acc = ref.int_matmul(A, B)
        for m in range(M):
            for n in range(N):
                assert acc[m, n] == sum(int(A[m, k]) * int(B[n, k]) for k in range(K))


def test_int_matmul_extreme_operands_exact():
    K = 12288
    A = np.full((2, K), 127, dtype=np.int64)
    A[1] = -127
    B = np.full((3, K), -127, dtype=np.int64)
    B[2, ::2] = 127
    acc = ref.int_matmul(A, B)
    assert acc[0, 0] == -127 * 127 * K and acc[1, 0] == 127 * 127 * K
    assert acc[0, 2] == 0
    assert abs(acc).max() < 2 ** 31


# ---------------------------------------------------------------- bf16 rounding
def test_to_bf16_matches_torch_on_fp32_values():
    rng = np.random.default_rng(7)
    y = np.concatenate([rng.standard_normal(20000) * 10.0 ** rng.integers(-6, 6, 20000),
                        [0.0, -0.0, 1.0, -3.0]]).astype(np.float32)
    want = torch.from_numpy(y).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(ref.to_bf16(y.astype(np.float64)), want)


def test_to_bf16_ties_to_even():
    assert ref.to_bf16(np.array([1 + 2 ** -8]))[0] == 1.0
    assert ref.to_bf16(np.array([1 + 3 * 2 ** -8]))[0] == 1 + 2 ** -6
    assert ref.to_bf16(np.array([-(1 + 2 ** -8)]))[0] == -1.0


# ---------------------------------------------------------------- end to end
def test_linear_one_hot_closed_form():
    # x = e_j and a single weight row e_j: x W^T = 1.  Both rotate to +-1/16
    # rows of H, quantise to +-127 codes, acc = 127^2 * 256 and
    # s_tok = s_row = (1/16)/127, so y = 1 exactly.
    x = np.zeros((1, 256))
    x[0, 77] = 1.0
    Wq, s_row, _ = ref.quantize_weight(x.copy())
    yb, aux = ref.linear_forward(x, Wq, s_row.astype(np.float64))
    assert aux["acc"][0, 0] == 127 * 127 * 256
    assert abs(aux["y64"][0, 0] - 1.0) < 1e-7
    assert yb[0, 0] == 1.0


def test_linear_against_float_product():
    rng = np.random.default_rng(8)
    x = rng.standard_normal((16, 512))
    W = rng.standard_normal((24, 512)) * 0.02
    Wq, s_row, _ = ref.quantize_weight(W)
    yb, aux = ref.linear_forward(x, Wq, s_row)
    exact = x @ W.T
    rel = np.linalg.norm(aux["y64"] - exact) / np.linalg.norm(exact)
    assert rel < 0.02   # two int8 roundings on Gaussian data


def test_rotation_lowers_error_with_outlier_channels():
    # the ConvRot claim ("Why ConvRot"): rotation spreads channel outliers so
    # per-token int8 rounding loses less
    import workloads
    x = workloads.activations(32, 512, outlier_count=4, outlier_scale=20.0).double().numpy()
    W = workloads.weight(256, 512).double().numpy()
    exact = x @ W.T
    errs = {}
    for group in (0, 256):
        Wq, s_row, _ = ref.quantize_weight(W, group)
        _, aux = ref.linear_forward(x, Wq, s_row, group=group)
        errs[group] = np.linalg.norm(aux["y64"] - exact) / np.linalg.norm(exact)
    assert errs[256] < 0.7 * errs[0]


# ---------------------------------------------------------------- RMSNorm / SmoothQuant
def test_rmsnorm_closed_forms():
    x = np.full((1, 256), 2.0)
    u = ref.rmsnorm(x, np.zeros(256), 0.0)
    assert np.allclose(u, 1.0, rtol=1e-15)
    # the norm multiplies by 1 + w, so w = -1 zeroes the output
    assert not ref.rmsnorm(x, -np.ones(256), 1e-6).any()
    rng = np.random.default_rng(9)
    x = rng.standard_normal((4, 512))
    u = ref.rmsnorm(x, np.zeros(512), 0.0)
    assert np.allclose(np.mean(u * u, axis=1), 1.0, rtol=1e-13)


def test_norm_codes_scale_invariant():
    rng = np.random.default_rng(10)
    x = rng.standard_normal((4, 512))
    w = rng.standard_normal(512) * 0.1
    q1, s1, _ = ref.rotate_quant_act(x, norm_w=w, eps=0.0)
    q2, s2, _ = ref.rotate_quant_act(x * 37.0, norm_w=w, eps=0.0)
    assert np.array_equal(q1, q2)
    assert np.allclose(s1, s2, rtol=1e-13)


def test_smoothquant_fold_preserves_the_linear():
    recipe = _golden("smoothquant_recipe.json")
    rng = np.random.default_rng(11)
    x = rng.standard_normal((32, 256)) * (1 + 20 * (rng.random(256) < 0.02))
    w = rng.standard_normal(256) * 0.1
    W = rng.standard_normal((16, 256)) * 0.02
    s, wf = ref.smoothquant_scales(x, w, 1e-6, W, alpha=recipe["alpha"])
    lhs = ref.rmsnorm(x, wf, 1e-6) @ (W * s[None, :]).T
    rhs = ref.rmsnorm(x, w, 1e-6) @ W.T
    assert np.max(np.abs(lhs - rhs)) < 1e-12 * np.max(np.abs(rhs)) * 100


def test_smoothquant_scale_closed_form():
    # one token, norm weight 0: the normalised activation of [4, -2, 0, 0...]
    # column 0 has max |a| = 4 / rms; weight column 0 max |W| = 1
    x = np.zeros((1, 4))
    x[0, :2] = [4.0, -2.0]
    rms = math.sqrt((16 + 4) / 4)
    W = np.array([[1.0, 0.25, 1.0, 0.0], [-0.5, 0.0, 2.0, 3.0]])
    s, wf = ref.smoothquant_scales(x, np.zeros(4), 0.0, W)
    assert s[0] == pytest.approx(math.sqrt(4 / rms) / math.sqrt(1.0), rel=1e-15)
    assert s[1] == pytest.approx(math.sqrt(2 / rms) / math.sqrt(0.25), rel=1e-15)
    assert s[2] == 1.0 and s[3] == 1.0          # zero activation column
    assert wf[0] == pytest.approx(1 / s[0] - 1, rel=1e-15)


# ---------------------------------------------------------------- int4 layout
def test_int4_pack_nibble_order_and_roundtrip():
    # every byte value decodes to (low, high) two's-complement nibbles
    allb = np.arange(256, dtype=np.uint8)[None, :]
    codes = ref.unpack_int4(allb)[0]
    for b in range(256):
        lo, hi = b & 0xF, b >> 4
        assert codes[2 * b] == (lo - 16 if lo >= 8 else lo)
        assert codes[2 * b + 1] == (hi - 16 if hi >= 8 else hi)
    assert np.array_equal(ref.pack_int4(codes[None, :]), allb)
    assert ref.pack_int4(np.array([[-1, -8]]))[0, 0] == 0x8F


def test_int4_clip_row_on_grid_picks_full_range():
    v = np.array([[7.0, -3.0, 2.0, 0.0, -7.0, 1.0, 5.0, -6.0]]) * 0.125
    out = ref.quantize_weight_w4(v, group=0)
    assert out["clip"][0] == 1.0 and out["err"][0] == 0.0
    assert np.array_equal(out["codes"][0], [7, -3, 2, 0, -7, 1, 5, -6])


def test_int4_clip_search_exact_rational_brute_force():
    # exact rational arithmetic over the 21 candidates decides the argmin
    rng = np.random.default_rng(12)
    for _ in range(20):
        v = rng.integers(-200, 201, size=8) / 16.0
        v[0] = 12.5
        out = ref.quantize_weight_w4(v[None, :], group=0)
        best = None
        amax = Fraction(max(abs(Fraction(t)) for t in v))
        for i in range(21):
            c = Fraction(80 + i, 100)
            s = c * amax / 7
            err = Fraction(0)
            for t in v:
                t = Fraction(t)
                r = t / s
                q = max(-7, min(7, round(r)))   # Fraction round() is half-even
                err += (t - s * q) ** 2
            if best is None or err < best[0]:
                best = (err, c)
        assert abs(out["clip"][0] - float(best[1])) < 1e-12
        assert abs(out["err"][0] - float(best[0])) <= 1e-12 * max(1.0, float(best[0]))


def test_int4_clip_never_worse_than_plain_absmax_and_scale_equivariant():
    rng = np.random.default_rng(13)
    W = rng.standard_normal((32, 512)) * 0.02
    out = ref.quantize_weight_w4(W)
    plain = ref.quantize_weight_w4(W, clip_lo=1.0, clip_hi=1.0, clip_steps=1)
    assert np.all(out["err"] <= plain["err"] * (1 + 1e-12))
    assert np.abs(out["codes"]).max() <= 7
    out2 = ref.quantize_weight_w4(W * 8.0)
    assert np.array_equal(out2["codes"], out["codes"])
    assert np.allclose(out2["s64"], 8.0 * out["s64"], rtol=1e-15)


def test_int4_row_error_plausible_against_card():
    # soft check only: the card's 11.4 % is on real weights
    card = _golden("int4_row_error.json")["mean_relative_row_error"]
    rng = np.random.default_rng(14)
    W = rng.standard_normal((64, 4096)) * 0.02
    out = ref.quantize_weight_w4(W)
    deq = out["codes"].astype(np.float64) * out["s64"][:, None]
    rel = np.linalg.norm(out["rotated"] - deq, axis=1) / np.linalg.norm(out["rotated"], axis=1)
    assert abs(rel.mean() - card) < 0.03


def test_zero_row_with_zero_eps_stays_zero():
    x = np.zeros((2, 256))
    x[1, 3] = 1.0
    q, s, v = ref.rotate_quant_act(x, norm_w=np.zeros(256), eps=0.0)
    assert s[0] == 0.0 and not q[0].any() and np.isfinite(v).all()
    assert s[1] > 0


# ---------------------------------------------------------------- MLP boundary
def test_silu_matches_library_logistic():
    from scipy.special import expit
    rng = np.random.default_rng(21)
    z = np.concatenate([rng.uniform(-40, 40, 4000), [0.0, 1e-300, -1e-300, 700.0, -700.0, -1e4]])
    want = z * expit(z)
    got = ref.silu(z)
    assert np.all(np.isfinite(got))
    assert np.max(np.abs(got - want) / np.maximum(np.abs(want), 1e-300)) < 1e-14
    assert ref.silu(np.array([0.0]))[0] == 0.0


def test_silu_odd_part_identity():
    # silu(z) - silu(-z) = z * (sigmoid(z) + sigmoid(-z)) = z for every z
    z = np.linspace(-30, 30, 2001)
    assert np.max(np.abs(ref.silu(z) - ref.silu(-z) - z)) < 1e-13
    # and the even part is z * tanh(z / 2) / ... : silu(z) + silu(-z) = z tanh(z/2)
    assert np.max(np.abs(ref.silu(z) + ref.silu(-z) - z * np.tanh(z / 2))) < 1e-12


def test_interleave_gate_up_brute_force():
    I, K, B = 48, 3, ref.SWIGLU_BLOCK
    Wg = np.arange(I * K).reshape(I, K)
    Wu = 1000 + np.arange(I * K).reshape(I, K)
    out = ref.interleave_gate_up(Wg, Wu)
    assert out.shape == (2 * I, K)
    for r in range(2 * I):
        blk, w = divmod(r, 2 * B)
        src = Wg if w < B else Wu
        assert np.array_equal(out[r], src[blk * B + (w % B)])
    # every source row appears exactly once
    seen = sorted(map(tuple, out.tolist()))
    assert seen == sorted(map(tuple, np.concatenate([Wg, Wu]).tolist()))
    with pytest.raises(ValueError):
        ref.interleave_gate_up(Wg[:40], Wu[:40])


def test_swiglu_linear_is_silu_of_gate_times_up():
    rng = np.random.default_rng(22)
    M, I, K = 5, 32, 64
    Xq = rng.integers(-127, 128, (M, K))
    Wg = rng.integers(-127, 128, (I, K))
    Wu = rng.integers(-127, 128, (I, K))
    s_tok = rng.uniform(1e-4, 1e-3, M)
    sg = rng.uniform(1e-4, 1e-3, I)
    su = rng.uniform(1e-4, 1e-3, I)
    hb, h, _ = ref.swiglu_linear(Xq, s_tok, ref.interleave_gate_up(Wg, Wu),
                                 ref.interleave_gate_up(sg, su))
    _, yg, _ = ref.int8_linear(Xq, s_tok, Wg, sg)
    _, yu, _ = ref.int8_linear(Xq, s_tok, Wu, su)
    np.testing.assert_array_equal(h, ref.silu(yg) * yu)
    np.testing.assert_array_equal(hb, ref.to_bf16(ref.silu(yg) * yu))
    # a zero up scale or a zero gate row gives exactly zero
    hb0, _, _ = ref.swiglu_linear(Xq, s_tok, ref.interleave_gate_up(Wg, Wu),
                                  ref.interleave_gate_up(sg, np.zeros(I)))
    assert not np.any(hb0)
    hb1, _, _ = ref.swiglu_linear(Xq, s_tok, ref.interleave_gate_up(np.zeros_like(Wg), Wu),
                                  ref.interleave_gate_up(sg, su))
    assert not np.any(hb1)


def test_smoothquant_scales_of_closed_form():
    a = np.array([[2.0, -8.0, 0.0], [1.0, 4.0, 0.0]])
    W = np.array([[0.5, 1.0, 3.0], [-2.0, 0.25, 1.0]])
    s = ref.smoothquant_scales_of(a, W, alpha=0.5)
    assert s[0] == pytest.approx(math.sqrt(2.0) / math.sqrt(2.0), rel=1e-15)
    assert s[1] == pytest.approx(math.sqrt(8.0) / math.sqrt(1.0), rel=1e-15)
    assert s[2] == 1.0                          # all-zero activation column
    # alpha = 1 moves everything into the weight: s = max |a|
    np.testing.assert_allclose(ref.smoothquant_scales_of(a, W, alpha=1.0)[:2], [2.0, 8.0], rtol=1e-15)
    # scaling one activation column by t scales its s by t^alpha
    a2 = a.copy()
    a2[:, 1] *= 9.0
    assert ref.smoothquant_scales_of(a2, W)[1] == pytest.approx(3.0 * s[1], rel=1e-14)


def test_down_proj_fold_into_up_rows_preserves_the_mlp():
    rng = np.random.default_rng(23)
    M, H, I = 8, 256, 256
    x = rng.standard_normal((M, H))
    Wg = rng.standard_normal((I, H)) * 0.05
    Wu = rng.standard_normal((I, H)) * 0.05
    Wd = rng.standard_normal((H, I)) * 0.05
    h = ref.silu(x @ Wg.T) * (x @ Wu.T)
    h[:, 7] *= 100.0                                 # an outlier channel of the down input
    s = ref.smoothquant_scales_of(h, Wd)
    assert np.argmax(s) == 7
    # (h / s) (Wd diag(s))^T == h Wd^T
    lhs = (h / s[None, :]) @ (Wd * s[None, :]).T
    rhs = h @ Wd.T
    assert np.max(np.abs(lhs - rhs)) < 1e-12 * np.max(np.abs(rhs)) * 100
    # dividing up's rows by s before quantisation leaves the codes and divides
    # the row scales: the fold can be applied to s_row
    q0, s0, _ = ref.quantize_weight(Wu)
    q1, s1, _ = ref.quantize_weight(Wu / s[:, None])
    np.testing.assert_array_equal(q0, q1)
    np.testing.assert_allclose(ref.fold_smooth_into_rows(s0, s), s1, rtol=2e-7)


# ---------------------------------------------------------------- weight-only path
def test_weight_only_equals_the_plain_linear_for_a_representable_weight():
    # W built from integer codes: W = (s * Wq) R, so the stored weight of W is
    # exactly (Wq, s) and the weight-only path gives x W^T in float64
    rng = np.random.default_rng(31)
    N, K = 12, 512
    Wq = rng.integers(-127, 128, (N, K)).astype(np.float64)
    Wq[:, 0] = 127  # a full-range code in every row
    s = rng.uniform(1e-3, 1e-2, N)
    W = ref.rotate_groups(Wq * s[:, None])      # R is symmetric and orthogonal
    q, s_row, _ = ref.quantize_weight(W)
    np.testing.assert_array_equal(q, Wq)
    x = rng.standard_normal((5, K))
    _, y = ref.weight_only_linear(ref.rotate_act(x), q, s_row)
    np.testing.assert_allclose(y, x @ W.T, rtol=1e-6, atol=1e-9)  # s_row is fp32


def test_weight_only_one_hot_code_closed_form():
    Xr = np.arange(12, dtype=np.float64).reshape(3, 4)
    Wq = np.zeros((2, 4))
    Wq[1, 2] = -3
    _, y = ref.weight_only_linear(Xr, Wq, np.array([5.0, 0.5]))
    np.testing.assert_array_equal(y, [[0, -3.0], [0, -9.0], [0, -15.0]])


def test_rotate_act_is_the_rotation_of_the_norm():
    rng = np.random.default_rng(32)
    x = rng.standard_normal((3, 256))
    w = rng.standard_normal(256) * 0.1
    v = ref.rotate_act(x, 256, w, 1e-6)
    # orthogonal rotation: row norms of the normalised input are kept
    np.testing.assert_allclose(np.linalg.norm(v, axis=1), np.linalg.norm(ref.rmsnorm(x, w, 1e-6), axis=1),
                               rtol=1e-13)
    assert np.array_equal(ref.rotate_act(x, 0), x)
