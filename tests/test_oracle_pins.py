"""Pins of the CPU oracle to facts that do not come from the oracle itself.

Each test checks the oracle against something the pages or the mathematics fix: worked examples the
pages print (fixtures under tests/golden, each with its source), closed forms at alpha = 0 and 1,
invariants of the quantiser, independent library routines (numpy int64 matmul, numpy max, torch's
bf16 rounding) and a rigorous error bound of the whole quantised chain against the exact fp64 product.
The tests are chosen so that a plausible slip in the oracle (a transposed operand, a dropped term, the
wrong exponent or tie rule, a wrong index) fails at least one of them.
"""
import numpy as np
import pytest
import torch

from conftest import num, read_golden
from post_quantization_calib_b200 import synth


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def bits_to_f64(h: np.ndarray) -> np.ndarray:
    return (h.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def rand_bf16(shape, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    return bf16_bits((torch.randn(*shape, generator=g) * scale).to(torch.bfloat16))


# --------------------------------------------------------------------------------------------
# bf16 rounding: torch's CPU conversion is an independent implementation of round-to-nearest-even.

def test_bf16_rounding_matches_torch(orc):
    g = torch.Generator().manual_seed(1)
    v = torch.randn(4000, generator=g, dtype=torch.float32) * 10.0 ** torch.randint(-6, 6, (4000,), generator=g)
    # exact ties: low 16 bits == 0x8000, with even and odd kept parts
    ties = np.array([0x3F808000, 0x3F818000, 0xBF808000, 0xBF818000, 0x7F7F8000], np.uint32).view(np.float32)
    allv = np.concatenate([v.numpy(), ties, np.array([0.0, -0.0, 1e-40, np.inf, -np.inf], np.float32)])
    ours = orc.f32_to_bf16(allv)
    ref = bf16_bits(torch.from_numpy(allv).to(torch.bfloat16))
    assert np.array_equal(ours, ref)


# --------------------------------------------------------------------------------------------
# Abs-max reductions ("06 -- SmoothQuant...", section 3; "Taming the Outliers...", System Architecture)

def test_absmax_matches_numpy_bruteforce(orc):
    a = rand_bf16((37, 48), 2, scale=3.0)
    ref = np.abs(bits_to_f64(a)).max(axis=0).astype(np.float32)
    assert np.array_equal(orc.calibrate_absmax(a), ref)


def test_absmax_strided_rows_and_running_max(orc):
    a = rand_bf16((20, 64), 3)
    sub = np.ascontiguousarray(a)  # full buffer, reduce only the first 40 columns with ld = 64
    rows, ld, cols = 20, 64, 40
    amax = np.zeros(cols, np.float32)
    orc.lib().orc_calibrate_absmax(sub.ctypes.data, rows, cols, ld, None, 1e-6, amax.ctypes.data, 0)
    ref = np.abs(bits_to_f64(a[:, :cols])).max(axis=0)
    assert np.array_equal(amax.astype(np.float64), ref)
    # running max over two batches equals the max over their concatenation
    b1, b2 = rand_bf16((9, 32), 4), rand_bf16((11, 32), 5, scale=2.0)
    m = orc.calibrate_absmax(b1)
    m = orc.calibrate_absmax(b2, amax=m, accumulate=True)
    assert np.array_equal(m, orc.calibrate_absmax(np.concatenate([b1, b2])))


def test_absmax_with_rmsnorm_against_fp64(orc):
    # rows of small magnitude so that eps = 1e-6 changes the result by tens of percent:
    # a dropped eps, a missing gamma or the mean over the wrong axis fails this.
    x = rand_bf16((16, 256), 6, scale=1e-3)
    gamma = (1.0 + 0.1 * np.random.default_rng(6).standard_normal(256)).astype(np.float32)
    eps = 1e-6
    got = orc.calibrate_absmax(x, norm_gamma=gamma, eps=eps).astype(np.float64)
    xf = bits_to_f64(x)
    y = xf / np.sqrt((xf ** 2).mean(axis=1, keepdims=True) + eps) * gamma.astype(np.float64)
    ref = np.abs(y).max(axis=0)
    assert np.allclose(got, ref, rtol=4e-7, atol=0)


# --------------------------------------------------------------------------------------------
# Smoothing factors: closed forms at the ends of the alpha range and the worked example.

def test_alpha_one_closed_form(orc):
    fx = read_golden("alpha_special_cases.txt")
    assert num(fx["alpha_one_smoothed_channel_max"]) == 1.0
    x = rand_bf16((64, 96), 7, scale=4.0)
    ax = orc.calibrate_absmax(x)
    aw = orc.calibrate_absmax(rand_bf16((80, 96), 8, scale=0.02))
    s, fold = orc.compute_scales(ax, aw, 1.0)
    assert np.array_equal(s, np.maximum(ax, np.float32(1e-5)))  # s_j = max|X_j|
    # every smoothed activation channel then peaks at exactly 1 (x / s in binary32)
    xs = bits_to_f64(x).astype(np.float32) / s[None, :]
    assert np.array_equal(np.abs(xs).max(axis=0), np.ones(96, np.float32))
    # and the folded reciprocal gives 1 to within one binary32 ulp
    assert np.all(np.abs(np.abs(bits_to_f64(x).astype(np.float32) * fold).max(axis=0) - 1.0) <= 2.0 ** -23)


def test_alpha_zero_closed_form(orc):
    fx = read_golden("alpha_special_cases.txt")
    assert num(fx["alpha_zero_smoothed_weight_max"]) == 1.0
    ax = orc.calibrate_absmax(rand_bf16((64, 96), 9, scale=4.0))
    w = rand_bf16((80, 96), 10, scale=0.02)
    aw = orc.calibrate_absmax(w)
    s, _ = orc.compute_scales(ax, aw, 0.0)
    # s_j = 1 / max|W_j|: correctly rounded reciprocal of the weight maximum
    ref = (1.0 / aw.astype(np.float64))
    assert np.all(np.abs(s.astype(np.float64) / ref - 1.0) <= 2.0 ** -24)
    # smoothed weight columns (diag(s) W) then peak at 1 within a binary32 ulp
    wmax = np.abs(bits_to_f64(w).astype(np.float32) * s[None, :]).max(axis=0)
    assert np.all(np.abs(wmax - 1.0) <= 2.0 ** -23)


def test_worked_example_s25(orc):
    fx = read_golden("outlier_channel_worked_example.txt")
    ax = np.array([num(fx["channel_absmax"])], np.float32)
    aw = np.array([num(fx["weight_absmax_derived"])], np.float32)
    s, fold = orc.compute_scales(ax, aw, num(fx["alpha"]))
    assert s[0] == np.float32(num(fx["s"]))
    # the outlier channel's range [-50, 50] becomes [-2, 2] ...
    chan = np.array([[-50.0], [50.0], [12.5]], np.float32)
    sm = np.abs(chan / s[None, :]).max()
    assert sm == num(fx["smoothed_absmax"])
    # ... and a per-tensor INT8 scale drops from 50/127 to 2/127
    assert np.isclose(50.0 / 127, num(fx["scale_before"])) and np.isclose(sm / 127, num(fx["scale_after"]))


def test_scales_floor_and_fold(orc):
    ax = np.array([0.0, 3.0, 7.5, 1e-9], np.float32)
    aw = np.array([0.5, 0.0, 0.1, 0.2], np.float32)
    gamma = np.array([1.1, 0.9, 1.0, 1.3], np.float32)
    s, fold = orc.compute_scales(ax, aw, 0.5, gamma)
    assert np.all(np.isfinite(s)) and np.all(s >= np.float32(1e-5))
    # fold times s gives back gamma to within one rounding
    assert np.allclose(fold.astype(np.float64) * s, gamma, rtol=2 ** -23, atol=0)
    s2, fold2 = orc.compute_scales(ax, aw, 0.5, None)
    assert np.array_equal(s, s2) and np.allclose(fold2.astype(np.float64) * s2, 1.0, rtol=2 ** -23)


def test_scale_exponent_is_one_minus_alpha(orc):
    # the variant with exponent alpha on the weight term would give s = (ax/aw)^alpha; at
    # alpha = 0.25, ax = 16, aw = 1/16: 16^0.25 / (1/16)^0.75 = 2 * 8 = 16, whereas the variant
    # gives (256)^0.25 = 4.
    s, _ = orc.compute_scales(np.array([16.0], np.float32), np.array([1.0 / 16], np.float32), 0.25)
    assert s[0] == 16.0


# --------------------------------------------------------------------------------------------
# Quantiser ("Taming the Outliers...", Why Outliers Break Quantization; tie rule: half away from 0)

def test_quantiser_tie_rule_and_range(orc):
    # one weight row with max 127 gives delta = 1 and 1/delta = 1 exactly, so the codes are the
    # rounded values themselves: ties go away from zero (half-to-even would give 2, -2, 0, 0).
    row = np.array([[2.5, -2.5, 0.5, -0.5, 1.5, 127.0, -126.5, 3.25]], np.float32)
    wq, ws = orc.smooth_quantize_weight(bf16_bits(torch.from_numpy(row).to(torch.bfloat16)))
    assert ws[0] == 1.0
    assert wq[0].tolist() == [3, -3, 1, -1, 2, 127, -127, 3]
    z, zs = orc.smooth_quantize_weight(np.zeros((2, 16), np.uint16))
    assert np.all(z == 0) and np.all(zs == 0)


def test_step_size_worked_example(orc):
    fx = read_golden("step_size_example.txt")
    for mkey, dkey, ckey in (("max_a", "delta_a", "code_a"), ("max_b", "delta_b", "code_b_arithmetic")):
        row = torch.tensor([[num(fx[mkey]), num(fx["value"])]], dtype=torch.float32).to(torch.bfloat16)
        wq, ws = orc.smooth_quantize_weight(bf16_bits(row))
        # the page prints the step to three significant digits
        assert abs(ws[0] - num(fx[dkey])) <= 1e-3 * num(fx[dkey])
        assert wq[0, 0] == 127 and wq[0, 1] == int(num(fx[ckey]))


def test_level_width_example(orc):
    fx = read_golden("level_width_example.txt")
    top = num(fx["tensor_max"])
    vals = np.concatenate([[top], np.linspace(-num(fx["median_channel_max"]), num(fx["median_channel_max"]), 501)])
    x = bf16_bits(torch.tensor(vals[None, :], dtype=torch.float32).to(torch.bfloat16))
    xq, xs = orc.rmsnorm_smooth_quant(x, np.ones(x.shape[1], np.float32), apply_norm=False)
    assert abs(2 * xs[0] * 127 / 255 - num(fx["level_width"])) < 0.005  # 255 levels over [-17.5, 17.5]
    levels = np.unique(xq[0, 1:])
    assert abs(len(levels) - num(fx["levels_about"])) <= 1


def test_six_channel_example(orc):
    fx = read_golden("six_channel_example.txt")
    v = np.array([float(t) for t in fx["vector"].split()], np.float32)
    j = int(num(fx["outlier_index_1based"])) - 1
    s = np.ones_like(v)
    s[j] = num(fx["s_outlier"])
    x = bf16_bits(torch.from_numpy(v[None, :]).to(torch.bfloat16))
    xq, xs = orc.rmsnorm_smooth_quant(x, (1.0 / s).astype(np.float32), apply_norm=False)
    # after smoothing the outlier channel is the row maximum, about 1.2 (8.7 is 8.6875 in bf16)
    assert xq[0, j] == 127
    assert abs(xs[0] * 127 - num(fx["smoothed_outlier"])) < 0.01


def test_quantiser_invariants_random(orc):
    x = rand_bf16((33, 200), 11, scale=2.0)
    fold = (0.5 + np.random.default_rng(11).random(200)).astype(np.float32)
    xq, xs = orc.rmsnorm_smooth_quant(x, fold, apply_norm=False)
    assert np.all(np.abs(xq).max(axis=1) == 127)            # the row maximum maps to +-127
    y = bits_to_f64(x) * fold.astype(np.float64)
    err = np.abs(xq * xs[:, None].astype(np.float64) - y)
    assert np.all(err <= xs[:, None] * (0.5 + 2e-5) + 4 * 2.0 ** -24 * np.abs(y))
    assert np.allclose(xs, np.abs(y).max(axis=1) / 127, rtol=3e-7, atol=0)


def _near_tie_row():
    """A row of binary32 values whose products with fl32(127/m) lie within a rounding of k + 1/2:
    y_k = fl32((k + 1/2) / fl32(127/m)) for k = 0..126, both signs, the row maximum m itself, zeros to 256."""
    m = np.float32(37.123)
    inv = np.float32(127.0) / m
    y = ((np.arange(127) + 0.5) / np.float64(inv)).astype(np.float32)
    row = np.zeros(256, np.float32)
    row[0], row[1:128], row[128:255] = m, y, -y
    return row, m, inv


def test_codes_round_the_exact_product(orc):
    """The INT8 code is round-half-away-from-zero of the exact product v * fl32(127/m), rounded once:
    checked element by element with exact rational arithmetic on values placed next to the ties
    k + 1/2, where rounding the product to binary32 first would move a third of them by one code.
    The values enter as the smoothing factors of a weight row of ones (w' = 1 * s = s exactly)."""
    from fractions import Fraction
    row, m, inv = _near_tie_row()
    ones = bf16_bits(torch.ones(1, 256, dtype=torch.bfloat16))
    wq, ws = orc.smooth_quantize_weight(ones, row)
    assert ws[0] == m / np.float32(127) and abs(int(wq[0, 0])) == 127

    def rha(fr):
        f = int(abs(fr) + Fraction(1, 2))         # floor(|p| + 1/2) for p >= 0
        return f if fr >= 0 else -f
    exact = np.array([rha(Fraction(float(v)) * Fraction(float(inv))) for v in row])
    assert np.array_equal(wq[0].astype(np.int64), np.clip(exact, -127, 127))
    twice = np.array([rha(Fraction(float(np.float32(np.float64(v) * np.float64(inv))))) for v in row])
    assert (twice != exact).sum() > 20                # the fixture does tell the two readings apart


def _tiny_rows(rows, K, seed):
    """bf16 rows whose largest magnitude lies between the bf16 subnormals and ~1e-37, where 127 / m
    (and 448 / m) overflows binary32; one row is all zero except one subnormal, one is all zero."""
    rng = np.random.default_rng(seed)
    mag = 2.0 ** rng.uniform(-133, -123, size=(rows, K))
    v = (mag * rng.choice([-1.0, 1.0], size=(rows, K))).astype(np.float32)
    v[1, :] = 0.0
    v[1, 3] = -2.0 ** -133                       # the smallest bf16 subnormal
    v[2, :] = 0.0
    v[3, 5] = 0.0
    return bf16_bits(torch.from_numpy(v).to(torch.bfloat16))


def test_tiny_rows_quantise_like_their_scaled_copies(orc):
    """A row whose maximum m is so small that 127 / m overflows binary32 is quantised as the same row
    scaled by a power of two into the normal range: the quantiser is scale-free, and a power-of-two
    scaling is exact in every step (so the codes must be identical), while the step is still
    fl(m / 127) of the unscaled m. Per-token (direct input), weight rows (s = 1) and FP8."""
    x = _tiny_rows(6, 64, 90)
    xf = bits_to_f64(x)
    one = np.ones(64, np.float32)
    big = bf16_bits(torch.from_numpy((xf * 2.0 ** 80).astype(np.float32)).to(torch.bfloat16))
    assert np.array_equal(bits_to_f64(big), xf * 2.0 ** 80)        # the scaling itself is exact
    q, d = orc.rmsnorm_smooth_quant(x, one, apply_norm=False)
    qb, db = orc.rmsnorm_smooth_quant(big, one, apply_norm=False)
    assert np.array_equal(q, qb)
    m = np.abs(xf).max(axis=1).astype(np.float32)
    assert np.array_equal(d, np.where(m > 0, m / np.float32(127), 0).astype(np.float32))
    nz = m > 0
    assert np.all(np.abs(q[nz]).max(axis=1) == 127) and np.all(q[~nz] == 0)
    # codes within half a level of the exact v / delta (exact rational arithmetic in binary64 is
    # exact here: the scaled values have 8 significant bits)
    t = xf[nz] * 2.0 ** 80 * 127 / (m[nz].astype(np.float64)[:, None] * 2.0 ** 80)
    assert np.all(np.abs(q[nz] - t) <= 0.5 + 1e-5)
    wq, ws = orc.smooth_quantize_weight(x)
    assert np.array_equal(wq, q) and np.array_equal(ws, d)
    f8, d8 = orc.rmsnorm_smooth_quant_f8(x, one, apply_norm=False)
    f8b, _ = orc.rmsnorm_smooth_quant_f8(big, one, apply_norm=False)
    assert np.array_equal(f8, f8b)
    assert np.array_equal(d8, np.where(m > 0, m / np.float32(448), 0).astype(np.float32))


def test_static_scale_with_overflowing_reciprocal(orc):
    """A static maximum below 127 / FLT_MAX: fl(127 / m) is +inf. Every nonzero value lies beyond the
    representable step and saturates at +-127; a zero value still codes 0 (not the NaN of 0 * inf)."""
    s2 = orc.static_scale(np.array([1e-38, 3e-38], np.float32))
    assert s2[0] == np.float32(3e-38) / np.float32(127) and np.isinf(s2[1])
    x = _tiny_rows(4, 32, 91)
    q, xs = orc.rmsnorm_smooth_quant_static(x, np.ones(32, np.float32), s2, apply_norm=False)
    xf = bits_to_f64(x)
    assert np.array_equal(q, (np.sign(xf) * 127).astype(np.int8))
    assert np.all(xs == s2[0])


def test_rmsnorm_constant_rows_and_scale_invariance(orc):
    K = 128
    x = np.zeros((3, K), np.float32)
    x[0] = 0.75
    x[1] = -3.0
    x[2, ::2] = 2.0
    x[2, 1::2] = -2.0
    xb = bf16_bits(torch.from_numpy(x).to(torch.bfloat16))
    xq, xs = orc.rmsnorm_smooth_quant(xb, np.ones(K, np.float32), eps=0.0, apply_norm=True)
    assert np.all(xq[0] == 127) and np.all(xq[1] == -127)
    assert np.all(xq[2, ::2] == 127) and np.all(xq[2, 1::2] == -127)
    assert np.allclose(xs, 1.0 / 127, rtol=2e-7)
    # doubling a row leaves its codes unchanged (RMSNorm is scale free; power-of-two scaling is exact)
    r = rand_bf16((4, K), 12)
    r2 = bf16_bits(torch.from_numpy(bits_to_f64(r).astype(np.float32) * 2).to(torch.bfloat16))
    f = (1 + 0.1 * np.random.default_rng(12).standard_normal(K)).astype(np.float32)
    assert np.array_equal(orc.rmsnorm_smooth_quant(r, f, eps=0.0)[0], orc.rmsnorm_smooth_quant(r2, f, eps=0.0)[0])


# --------------------------------------------------------------------------------------------
# Static per-tensor activation scale ("SmoothQuant and W8A8...", "One layer, measured" and
# "Gotchas"): one scale from the calibration maximum, values past it clipped. Pinned against the
# per-token quantiser (pinned above) through relations that hold exactly.

@pytest.mark.parametrize("norm", [False, True])
def test_static_scale_equals_dynamic_on_its_own_calibration_token(orc, norm):
    # calibrating on a single token and quantising that token gives the per-token result exactly
    K = 96
    fold = (0.5 + np.random.default_rng(21).random(K)).astype(np.float32)
    for seed in range(5):
        x = rand_bf16((1, K), 40 + seed, scale=3.0)
        amax_y = orc.calibrate_absmax(x, norm_gamma=fold if norm else None, eps=1e-6)
        if not norm:
            amax_y = (amax_y * fold).astype(np.float32)    # exact: one binary32 product per channel
        s2 = orc.static_scale(amax_y)
        q_s, xs_s = orc.rmsnorm_smooth_quant_static(x, fold, s2, eps=1e-6, apply_norm=norm)
        q_d, xs_d = orc.rmsnorm_smooth_quant(x, fold, eps=1e-6, apply_norm=norm)
        assert np.array_equal(q_s, q_d) and np.array_equal(xs_s, xs_d)


def test_static_step_is_the_largest_per_token_step(orc):
    # delta = m / 127 is monotone in m, and m is the largest row maximum of the calibration set
    K = 200
    x = rand_bf16((64, K), 50, scale=2.0)
    fold = (0.25 + np.random.default_rng(50).random(K)).astype(np.float32)
    amax_y = orc.calibrate_absmax(x, norm_gamma=fold, eps=1e-6)
    s2 = orc.static_scale(amax_y)
    _, xs_d = orc.rmsnorm_smooth_quant(x, fold, eps=1e-6, apply_norm=True)
    assert s2[0] == xs_d.max()
    assert s2[1] == np.float32(127) / amax_y.max()          # numpy binary32 division: one IEEE rounding


def test_static_codes_clip_and_stay_within_half_a_step(orc):
    K = 64
    scale2 = np.array([np.float32(2.0) / np.float32(127), np.float32(127) / np.float32(2.0)], np.float32)
    fold = np.ones(K, np.float32)
    v = np.linspace(-6.0, 6.0, K).astype(np.float32)        # the calibrated maximum is 2
    x = bf16_bits(torch.from_numpy(v[None, :]).to(torch.bfloat16))
    q, xs = orc.rmsnorm_smooth_quant_static(x, fold, scale2, apply_norm=False)
    y = bits_to_f64(x)[0]
    assert np.all(q[0][y >= 2.0] == 127) and np.all(q[0][y <= -2.0] == -127)
    inside = np.abs(y) < 2.0
    assert np.all(np.abs(q[0][inside] * float(scale2[0]) - y[inside]) <= float(scale2[0]) * (0.5 + 1e-5))
    assert np.all(xs == scale2[0])
    z = orc.static_scale(np.zeros(8, np.float32))
    assert z[0] == 0 and z[1] == 0
    qz, xz = orc.rmsnorm_smooth_quant_static(x, fold, z, apply_norm=False)
    assert not qz.any() and not xz.any()


# --------------------------------------------------------------------------------------------
# Fold into the previous linear's output columns ("06 -- SmoothQuant...", section 7): with powers
# of two the fold is exact and the chain is unchanged; otherwise each weight is within half a bf16
# step of w / s.

def test_fold_into_prev_linear_power_of_two_is_exact(orc):
    K, Kp, N = 64, 48, 40
    g = torch.Generator().manual_seed(60)
    w_prev = bf16_bits((torch.randn(K, Kp, generator=g) * 0.05).to(torch.bfloat16))
    b_prev = bf16_bits((torch.randn(K, generator=g) * 0.05).to(torch.bfloat16))
    s = (2.0 ** torch.randint(-4, 5, (K,), generator=g).double()).numpy().astype(np.float32)
    fold = (np.float32(1) / s).astype(np.float32)
    wo, bo = orc.fold_into_prev_linear(w_prev, b_prev, fold)
    assert np.array_equal(bits_to_f64(wo), bits_to_f64(w_prev) / s[:, None].astype(np.float64))
    assert np.array_equal(bits_to_f64(bo), bits_to_f64(b_prev) / s.astype(np.float64))
    # the method's invariance: (h W_prev^T + b) diag(1/s) diag(s) W^T = (h W_prev^T + b) W^T
    h = torch.randn(7, Kp, generator=g).double().numpy()
    w = torch.randn(N, K, generator=g).double().numpy()
    y_prev = h @ bits_to_f64(w_prev).T + bits_to_f64(b_prev)
    y_fold = h @ bits_to_f64(wo).T + bits_to_f64(bo)
    assert np.allclose((y_fold * s) @ w.T, y_prev @ w.T, rtol=1e-12, atol=1e-12)


def test_fold_into_prev_linear_rounding_and_w_scale(orc):
    K, Kp = 32, 40
    g = torch.Generator().manual_seed(61)
    w_prev = bf16_bits(torch.randn(K, Kp, generator=g).to(torch.bfloat16))
    fold = (0.3 + np.random.default_rng(61).random(K)).astype(np.float32)
    wo, bo = orc.fold_into_prev_linear(w_prev, None, fold)
    assert bo is None
    exact = bits_to_f64(w_prev) * fold[:, None].astype(np.float64)
    assert np.all(np.abs(bits_to_f64(wo) - exact) <= np.abs(exact) * 2.0 ** -8 + 1e-30)
    ws = (np.random.default_rng(62).random(K) * 1e-2).astype(np.float32)
    assert np.array_equal(orc.fold_into_w_scale(ws, fold), ws * fold)     # one binary32 product each


@pytest.mark.parametrize("pow2", [True, False])
def test_fold_into_w_scale_divides_the_int8_layer_output_by_s(orc, pow2):
    """"06 -- SmoothQuant...", section 7: folding 1/s into an INT8 previous layer must make that layer's
    dequantised output arrive divided by s, column by column. The previous layer's output is taken
    through the oracle's own INT8 GEMM and dequantisation, once with the folded scale and once
    without: with power-of-two s every step scales exactly (bit-exact bf16 outputs); otherwise the
    folded scale is the exact ws / s within two binary32 roundings (fl(1/s), then the product), and the
    bf16 outputs agree within one bf16 rounding of that."""
    T, K, Kp = 24, 40, 64                  # previous layer: [T, Kp] x [K, Kp]^T -> [T, K]
    rng = np.random.default_rng(63)
    xq = rng.integers(-127, 128, size=(T, Kp), dtype=np.int8)
    wq = rng.integers(-127, 128, size=(K, Kp), dtype=np.int8)
    xs = (rng.random(T) * 1e-2 + 1e-3).astype(np.float32)
    ws = (rng.random(K) * 1e-2 + 1e-3).astype(np.float32)
    if pow2:
        s = (2.0 ** rng.integers(-6, 7, size=K)).astype(np.float32)
    else:
        s = (0.05 + 20 * rng.random(K)).astype(np.float32)
    fold = (np.float32(1.0) / s).astype(np.float32)               # fl32(1/s): the fold without gamma
    ws_f = orc.fold_into_w_scale(ws, fold)
    rel = np.abs(ws_f.astype(np.float64) * s.astype(np.float64) / ws.astype(np.float64) - 1.0)
    assert np.all(rel <= 2.0 ** -23 + 2.0 ** -46), "folded scale is not ws / s within two roundings"
    y0, acc = orc.w8a8_linear(xq, xs, wq, ws)                      # unfolded layer (bf16 bits)
    y1, acc1 = orc.w8a8_linear(xq, xs, wq, ws_f)                   # folded layer
    assert np.array_equal(acc, acc1)
    v0, v1 = bits_to_f64(y0), bits_to_f64(y1)
    target = v0 / s[None, :].astype(np.float64)
    if pow2:
        assert np.array_equal(v1, target), "a power-of-two fold must divide the output exactly"
    else:
        # |y1 - y0 / s| <= bf16 rounding of both outputs plus the scale's two binary32 roundings
        tol = (np.abs(target) + np.abs(v1)) * (2.0 ** -8 + 2.0 ** -22) + 1e-30
        assert np.all(np.abs(v1 - target) <= tol)
    # a wrong index (the fold applied to the wrong channel) moves some output column by far more
    wrong = orc.fold_into_w_scale(ws, np.roll(fold, 1))
    yw, _ = orc.w8a8_linear(xq, xs, wq, wrong)
    assert not np.allclose(bits_to_f64(yw), target, rtol=1e-2)


# --------------------------------------------------------------------------------------------
# LayerNorm fold ("SmoothQuant: Weight-Only vs W8A8", "Integration with Transformers": S^-1 into the
# LayerNorm's gamma and beta): the oracle's LayerNorm against numpy binary64, scale freedom, constant rows, and the fold
# giving y / s.

def _ln64(x64, g, b, eps):
    mu = x64.mean(axis=1, keepdims=True)
    c = x64 - mu
    return c / np.sqrt((c * c).mean(axis=1, keepdims=True) + eps) * g + b, mu


def test_layernorm_calibration_against_fp64(orc):
    x = rand_bf16((40, 128), 80, scale=2.0)
    x64 = bits_to_f64(x) + 0.0
    g = (1 + 0.1 * np.random.default_rng(80).standard_normal(128)).astype(np.float32)
    b = (0.05 * np.random.default_rng(81).standard_normal(128)).astype(np.float32)
    amax = orc.calibrate_absmax_layernorm(x, g, b, eps=1e-5)
    y64, mu = _ln64(x64, g.astype(np.float64), b.astype(np.float64), 1e-5)
    ref = np.abs(y64).max(axis=0)
    assert np.all(np.abs(amax - ref) <= 16 * 2.0 ** -24 * (ref + np.abs(b)) + 4 * 2.0 ** -24 * np.abs(mu).max() * np.abs(g) * 10)
    # running maximum over two batches equals the maximum over their concatenation
    a2 = orc.calibrate_absmax_layernorm(x[20:], g, b, eps=1e-5, amax=orc.calibrate_absmax_layernorm(x[:20], g, b, eps=1e-5).copy(),
                                        accumulate=True)
    assert np.array_equal(a2, amax)


def test_layernorm_quant_fold_and_invariances(orc):
    K = 96
    x = rand_bf16((12, K), 82, scale=1.5)
    rng = np.random.default_rng(82)
    g = (1 + 0.1 * rng.standard_normal(K)).astype(np.float32)
    b = (0.1 * rng.standard_normal(K)).astype(np.float32)
    s = (0.5 + rng.random(K) * 4).astype(np.float32)
    fold = (g / s).astype(np.float32)
    bf = orc.fold_layernorm_bias(b, s)
    assert np.array_equal(bf, (b / s).astype(np.float32))
    xq, xs = orc.layernorm_smooth_quant(x, fold, bf, eps=1e-5)
    y64, _ = _ln64(bits_to_f64(x), g.astype(np.float64), b.astype(np.float64), 1e-5)
    t = y64 / s.astype(np.float64)                           # the smoothed activation the codes stand for
    err = np.abs(xq * xs[:, None].astype(np.float64) - t)
    assert np.all(err <= xs[:, None] * (0.5 + 1e-4) + 1e-6 * np.abs(t))
    assert np.all(np.abs(xq).max(axis=1) == 127)
    # doubling a row (exact) leaves LayerNorm, so the codes, unchanged
    x2 = bf16_bits(torch.from_numpy(bits_to_f64(x).astype(np.float32) * 2).to(torch.bfloat16))
    assert np.array_equal(orc.layernorm_smooth_quant(x2, fold, bf, eps=0.0)[0], orc.layernorm_smooth_quant(x, fold, bf, eps=0.0)[0])
    # a constant row normalises to zero: what remains is the folded bias
    c = bf16_bits(torch.full((1, K), 0.75).to(torch.bfloat16))
    qc, sc = orc.layernorm_smooth_quant(c, fold, bf, eps=1e-5)
    qb, sb = orc.rmsnorm_smooth_quant(bf16_bits(torch.ones(1, K).to(torch.bfloat16)), bf, apply_norm=False)
    assert np.array_equal(qc, qb) and np.array_equal(sc, sb)


# --------------------------------------------------------------------------------------------
# FP8 E4M3 variant ("SmoothQuant and W8A8...", "One layer, measured"): torch's float8_e4m3fn type
# is the independent check of the format (decode of every finite code, round-to-nearest-even
# encode including exact ties and subnormals); saturation at 448 is the closed form.

def _finite_e4m3_codes():
    c = np.arange(256, dtype=np.uint8)
    return c[(c & 0x7F) != 0x7F]


def test_e4m3_decode_matches_torch(orc):
    c = _finite_e4m3_codes()
    ref = torch.from_numpy(c.copy()).view(torch.float8_e4m3fn).float().numpy()
    assert np.array_equal(orc.e4m3_decode(c), ref)
    assert orc.e4m3_decode(np.uint8(0x7E)) == 448.0 and orc.e4m3_decode(np.uint8(0x01)) == 2.0 ** -9


def test_e4m3_encode_matches_torch_and_saturates(orc):
    ref = torch.from_numpy(_finite_e4m3_codes().copy()).view(torch.float8_e4m3fn).float().numpy()
    pos = np.sort(ref[ref > 0])
    rng = np.random.default_rng(70)
    vals = np.concatenate([ref, (pos[:-1] + pos[1:]) / 2, -(pos[:-1] + pos[1:]) / 2,   # every exact tie
                           rng.uniform(-448, 448, 4000), rng.standard_normal(4000) * 2.0 ** -8]).astype(np.float32)
    tref = torch.from_numpy(vals).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(orc.e4m3_encode(vals), tref)
    assert np.all(orc.e4m3_encode(np.array([448.5, 470.0, 1e9], np.float32)) == 0x7E)
    assert np.all(orc.e4m3_encode(np.array([-448.5, -1e9], np.float32)) == 0xFE)


def test_fp8_quantiser_invariants(orc):
    x = rand_bf16((17, 256), 71, scale=3.0)
    fold = (0.5 + np.random.default_rng(71).random(256)).astype(np.float32)
    xq, xs = orc.rmsnorm_smooth_quant_f8(x, fold, apply_norm=True)
    assert np.all((xq & 0x7F).max(axis=1) == 0x7E)               # the row maximum maps to +-448
    wq, ws = orc.smooth_quantize_weight_f8(rand_bf16((9, 256), 72), fold)
    assert np.all((wq & 0x7F).max(axis=1) == 0x7E)
    y = bits_to_f64(x) * fold.astype(np.float64)                 # without the norm: y = x * fold
    xq2, xs2 = orc.rmsnorm_smooth_quant_f8(x, fold, apply_norm=False)
    t = y / xs2[:, None].astype(np.float64)                       # the value each code stands for
    d = orc.e4m3_decode(xq2).astype(np.float64)
    normal = np.abs(d) >= 2.0 ** -6
    assert np.all(np.abs(d - t)[normal] <= np.abs(t)[normal] * 2.0 ** -4 * (1 + 1e-6))   # half a step of 3 bits
    assert np.all(np.abs(d - t)[~normal] <= 2.0 ** -10 * (1 + 1e-6) + np.abs(t)[~normal] * 2.0 ** -20)


def test_fp8_gemm_exact_and_dequant(orc):
    rng = np.random.default_rng(73)
    c = _finite_e4m3_codes()
    xq = rng.choice(c, size=(11, 700)).astype(np.uint8)
    wq = rng.choice(c, size=(13, 700)).astype(np.uint8)
    dx = torch.from_numpy(xq).view(torch.float8_e4m3fn).double().numpy()
    dw = torch.from_numpy(wq).view(torch.float8_e4m3fn).double().numpy()
    acc = orc.gemm_f8(xq, wq)
    assert np.array_equal(acc, dx @ dw.T)                       # both exact: every partial sum is representable
    xs = (rng.random(11) * 1e-2).astype(np.float32)
    ws = (rng.random(13) * 1e-2).astype(np.float32)
    y, _ = orc.w8a8_linear_f8(xq, xs, wq, ws)
    exact = acc * xs[:, None].astype(np.float64) * ws[None, :].astype(np.float64)
    assert np.all(np.abs(bits_to_f64(y) - exact) <= np.abs(exact) * (2.0 ** -8 + 2.0 ** -22) + 1e-30)


# --------------------------------------------------------------------------------------------
# INT8 GEMM ("06 -- SmoothQuant...", section 7): numpy int64 matmul is the independent check.

def test_gemm_matches_numpy_int64(orc):
    rng = np.random.default_rng(13)
    xq = rng.integers(-127, 128, (29, 160), dtype=np.int8)
    wq = rng.integers(-127, 128, (41, 160), dtype=np.int8)
    ref = xq.astype(np.int64) @ wq.astype(np.int64).T
    assert np.array_equal(orc.gemm_s8(xq, wq), ref)
    rows, cols = np.array([28, 0, 5]), np.array([40, 3])
    assert np.array_equal(orc.gemm_s8(xq, wq, rows, cols), ref[np.ix_(rows, cols)])


def test_gemm_extreme_codes(orc):
    K = 8192
    xq = np.full((2, K), 127, np.int8)
    xq[1] = -127
    wq = np.full((3, K), -127, np.int8)
    wq[1] = 127
    wq[2, ::2] = 127
    acc = orc.gemm_s8(xq, wq)
    assert acc.tolist() == [[-K * 16129, K * 16129, 0], [K * 16129, -K * 16129, 0]]


# --------------------------------------------------------------------------------------------
# Dequant epilogue: against the exact fp64 value within one bf16 rounding.

def test_dequant_against_fp64(orc):
    rng = np.random.default_rng(14)
    acc = rng.integers(-2 ** 27, 2 ** 27, (17, 23)).astype(np.int32)
    xs = (rng.random(17) * 0.1).astype(np.float32)
    ws = (rng.random(23) * 0.001).astype(np.float32)
    bias = bf16_bits(torch.from_numpy(rng.standard_normal(23).astype(np.float32) * 0.02).to(torch.bfloat16))
    y = bits_to_f64(orc.dequant(acc, xs, ws, bias))
    ref = acc.astype(np.float64) * xs[:, None].astype(np.float64) * ws[None, :] + bits_to_f64(bias)[None, :]
    assert np.all(np.abs(y - ref) <= 2.0 ** -8 * np.abs(ref) + 1e-6 * (np.abs(acc) * xs[:, None] * ws[None, :]) + 1e-30)
    # zero accumulators give the bias exactly; no bias gives exact zeros
    z = orc.dequant(np.zeros((2, 23), np.int32), xs[:2], ws, bias)
    assert np.array_equal(z, np.broadcast_to(bias, (2, 23)))
    assert np.all(bits_to_f64(orc.dequant(np.zeros((2, 23), np.int32), xs[:2], ws)) == 0)


# --------------------------------------------------------------------------------------------
# The whole chain: quantised smoothed linear vs the exact fp64 product, within the rigorous bound
# implied by the two quantisers (half a step each, plus binary32 roundings). Also checks the
# invariance Y = (X diag(s)^-1)(diag(s) W) that lets the smoothed product stand for X W.

def _chain_bound_check(orc, x, w, gamma, bias, alpha, eps, apply_norm):
    T, K = x.shape
    ax = orc.calibrate_absmax(x, norm_gamma=gamma if apply_norm else None, eps=eps)
    aw = orc.calibrate_absmax(w)
    s, fold = orc.compute_scales(ax, aw, alpha, gamma if apply_norm else None)
    wq, ws = orc.smooth_quantize_weight(w, s)
    xq, xs = orc.rmsnorm_smooth_quant(x, fold, eps=eps, apply_norm=apply_norm)
    y, acc = orc.w8a8_linear(xq, xs, wq, ws, bias)

    xf, wf = bits_to_f64(x), bits_to_f64(w)
    if apply_norm:
        xin = xf / np.sqrt((xf ** 2).mean(axis=1, keepdims=True) + eps) * gamma.astype(np.float64)
    else:
        xin = xf
    b = bits_to_f64(bias) if bias is not None else np.zeros(w.shape[0])
    exact = xin @ wf.T + b
    sd = s.astype(np.float64)
    xhat, what = xin / sd, wf * sd            # smoothed operands in exact arithmetic
    assert np.allclose(xhat @ what.T + b, exact, rtol=1e-12, atol=1e-12)   # invariance, fp64

    ea = xs[:, None] * (0.5 + 2e-5) + 6 * 2.0 ** -24 * np.abs(xhat)     # [T, K]
    eb = ws[:, None] * (0.5 + 2e-5) + 2 * 2.0 ** -24 * np.abs(what)     # [N, K]
    bound = ea @ np.abs(what).T + np.abs(xhat) @ eb.T + ea @ eb.T
    yq = acc.astype(np.float64) * xs[:, None] * ws[None, :] + b
    assert np.all(np.abs(yq - exact) <= bound * (1 + 1e-9) + 1e-12)
    yo = bits_to_f64(y)
    assert np.all(np.abs(yo - yq) <= 2.0 ** -8 * np.abs(yq) + 1e-6 * np.abs(yq) + 1e-30)
    return exact, yo


def test_chain_error_bound_no_norm(orc):
    w_ = synth.WORKLOADS[0]
    K, N, T = 256, 96, 40
    ch = synth.outlier_channels(K, synth.OutlierSpec(6, 50.0, 50.0), 21)
    x = bf16_bits(synth.outlier_tokens(T, K, ch, 22))
    w = bf16_bits(synth.normal_weight(N, K, 23))
    bias = bf16_bits(synth.bias_vector(N, 24))
    _chain_bound_check(orc, x, w, None, bias, w_.alpha, 1e-6, False)


def test_chain_error_bound_with_norm(orc):
    K, N, T = 256, 80, 33
    ch = synth.outlier_channels(K, synth.OutlierSpec(5, 10.0, 100.0), 31)
    x = bf16_bits(synth.outlier_tokens(T, K, ch, 32))
    w = bf16_bits(synth.normal_weight(N, K, 33))
    gamma = synth.norm_gamma(K, 34).numpy()
    _chain_bound_check(orc, x, w, gamma, None, 0.5, 1e-6, True)


def test_taming_simulation_per_tensor(orc):
    # "Taming the Outliers: A Deep Dive into SmoothQuant for LLM Quantization", "Implementation" (the
    # SmoothQuantLinear simulation): 128 input features, 64 outputs, 5 % of the channels scaled by 50,
    # 100 calibration and 10 test samples, alpha 0.5, per-tensor symmetric quantisation of both the
    # activations and the weight; the page prints the smoothed and the unsmoothed MSE against the
    # unquantised product and states that smoothing lowers it. Restated with the oracle's quantisers:
    # one per-tensor scale for x / s (from the test tokens' own maximum) and one for diag(s) W.
    K, N = 128, 64
    ch = synth.outlier_channels(K, synth.OutlierSpec(int(K * 0.05), 50.0, 50.0), 61)
    x_cal = bf16_bits(synth.outlier_tokens(100, K, ch, 62))
    x = bf16_bits(synth.outlier_tokens(10, K, ch, 63))
    w = bf16_bits(synth.normal_weight(N, K, 64, std=1.0))
    exact = bits_to_f64(x) @ bits_to_f64(w).T

    def mse(s):
        f_x = (1.0 / s).astype(np.float32) if s is not None else np.ones(K, np.float32)
        f_w = s.astype(np.float32) if s is not None else np.ones(K, np.float32)
        sx = orc.static_scale((orc.calibrate_absmax(x) * np.abs(f_x)).astype(np.float32))
        sw = orc.static_scale((orc.calibrate_absmax(w) * np.abs(f_w)).astype(np.float32))
        xq, xs = orc.rmsnorm_smooth_quant_static(x, f_x, sx, apply_norm=False)
        wq, ws = orc.rmsnorm_smooth_quant_static(w, f_w, sw, apply_norm=False)
        acc = orc.gemm_s8(xq, wq).astype(np.float64)
        y = acc * xs.astype(np.float64)[:, None] * ws.astype(np.float64)[None, :]
        return float(np.mean((y - exact) ** 2))

    s, _ = orc.compute_scales(orc.calibrate_absmax(x_cal), orc.calibrate_absmax(w), 0.5)
    base, smooth = mse(None), mse(s)
    assert smooth < 0.5 * base, (base, smooth)


def test_smoothing_reduces_error_on_outlier_data(orc):
    # qualitative claim of the pages ("SmoothQuant and W8A8...", One layer, measured; the MSE
    # comparison of "Taming the Outliers..."): on outlier-shaped data the smoothed W8A8 output is
    # closer to the exact product than the unsmoothed one.
    K, N, T = 512, 128, 64
    ch = synth.outlier_channels(K, synth.OutlierSpec(16, 10.0, 25.0, pinned=25.0), 41)
    x = bf16_bits(synth.outlier_tokens(T, K, ch, 42))
    w = bf16_bits(synth.normal_weight(N, K, 43))
    exact = bits_to_f64(x) @ bits_to_f64(w).T

    def err(s):
        fold = (1.0 / s).astype(np.float32) if s is not None else np.ones(K, np.float32)
        wq, ws = orc.smooth_quantize_weight(w, s)
        xq, xs = orc.rmsnorm_smooth_quant(x, fold, apply_norm=False)
        y, _ = orc.w8a8_linear(xq, xs, wq, ws)
        return np.linalg.norm(bits_to_f64(y) - exact) / np.linalg.norm(exact)

    s, _ = orc.compute_scales(orc.calibrate_absmax(x), orc.calibrate_absmax(w), 0.5)
    assert err(s) < 0.7 * err(None)


def test_alpha_sweet_spot_and_traps(orc):
    # The alpha sweep of "SmoothQuant and W8A8: Quantizing Activations Too", One layer, measured
    # (weights per output channel, activations on one static per-tensor scale from the calibration
    # maximum): alpha has a best middle range and two traps. Too small an alpha rescales channels by
    # their weights' range rather than flattening the activations, which is worse than no smoothing
    # when the outlier channels also carry the larger weights (built here: 2x weights there); too
    # large an alpha moves the range into the weights, whose quantisation error then dominates.
    K, N, T = 512, 128, 256
    ch = synth.outlier_channels(K, synth.OutlierSpec(16, 10.0, 25.0, pinned=25.0), 41)
    x = bf16_bits(synth.outlier_tokens(T, K, ch, 42))
    wt = synth.normal_weight(N, K, 43).float()
    wt[:, ch[0]] *= 2.0
    w = bf16_bits(wt.to(torch.bfloat16))
    exact = bits_to_f64(x) @ bits_to_f64(w).T
    ax, aw = orc.calibrate_absmax(x), orc.calibrate_absmax(w)

    def err(alpha):
        if alpha is None:
            s, fold = None, np.ones(K, np.float32)
        else:
            s, _ = orc.compute_scales(ax, aw, alpha)
            fold = (np.float32(1.0) / s).astype(np.float32)
        wq, ws = orc.smooth_quantize_weight(w, s)
        amax_y = (ax * fold).astype(np.float32)     # max |x * f| = fl(max |x| * f), rounding being monotone
        xq, xs = orc.rmsnorm_smooth_quant_static(x, fold, orc.static_scale(amax_y), apply_norm=False)
        y, _ = orc.w8a8_linear(xq, xs, wq, ws)
        return np.linalg.norm(bits_to_f64(y) - exact) / np.linalg.norm(exact)

    none, low, mid, high = err(None), err(0.1), err(0.7), err(1.0)
    assert mid < 0.5 * none            # the sweet spot
    assert low > none                  # too little: worse than no smoothing
    assert high > 2.0 * mid            # too much: the weights' error takes over
