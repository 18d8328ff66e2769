"""Pins of the CPU oracle against facts fixed by the pages and by mathematics (no GPU needed).

Each test checks the oracle against something other than itself: exact rational arithmetic, brute force
over all 16 levels, closed forms, an independent multiprecision library (mpmath), hand-worked examples
and invariants the AWQ pages state (the scaling identity of section 一 of the gsyq.cn AWQ page, ratio 0
reducing to plain round-to-nearest, the noise rule of section 2.1 of the hncyxsy.com outlier page).
"""
from decimal import Decimal, localcontext
from fractions import Fraction

import mpmath
import numpy as np
import pytest
import torch

from oracle import awq_oracle as orc
from weight_only_quantization_act_b200 import inputs

F32 = np.float32


def nearest_f32_of_fraction(v: Fraction) -> np.float32:
    """The float32 nearest to an exact rational (ties to even), found by exact comparison."""
    f = F32(float(v))
    cands = [np.nextafter(f, F32(-np.inf)), f, np.nextafter(f, F32(np.inf))]
    best = None
    for c in cands:
        d = abs(Fraction(float(c)) - v)
        if best is None or d < best[0] or (d == best[0] and int(c.view(np.uint32)) % 2 == 0):
            best = (d, c)
    return F32(best[1])


def midpoints(y: np.float32):
    lo = np.nextafter(y, F32(-np.inf))
    hi = np.nextafter(y, F32(np.inf))
    return (Fraction(float(lo)) + Fraction(float(y))) / 2, (Fraction(float(y)) + Fraction(float(hi))) / 2


# ------------------------------------------------------------------------------------------------ a1
def test_act_mean_matches_exact_rational_mean_tiny_workload():
    X, _, _ = inputs.make_inputs(inputs.workload(1))
    got = orc.act_mean(X)
    xf = inputs.bf16_bits_to_f32(X)
    N, K = X.shape
    bad = []
    for k in range(K):
        exact = sum(Fraction(float(abs(v))) for v in xf[:, k]) / N
        if nearest_f32_of_fraction(exact) != got[k]:
            bad.append(k)
    assert not bad, f"columns whose fp64 ordered mean does not round like the exact mean: {bad}"


def test_act_mean_single_row_and_constant_column():
    rng = np.random.default_rng(3)
    row = inputs.f32_to_bf16_bits(rng.standard_normal((1, 384)).astype(F32))
    assert np.array_equal(orc.act_mean(row), np.abs(inputs.bf16_bits_to_f32(row[0])))
    col = np.full((1000, 128), inputs.f32_to_bf16_bits(np.array([-0.375], F32))[0], np.uint16)
    assert np.all(orc.act_mean(col) == F32(0.375))


def test_act_mean_takes_absolute_values_per_column():
    x = np.zeros((3, 128), F32)
    x[:, 5] = [-1.0, 2.0, -3.0]
    x[:, 7] = [4.0, -4.0, 4.0]
    got = orc.act_mean(inputs.f32_to_bf16_bits(x))
    assert got[5] == F32(2.0) and got[7] == F32(4.0)
    assert np.count_nonzero(got) == 2


# ------------------------------------------------------------------------------------------------ a2
def test_ratio_grid_is_nearest_fp32_of_j_over_n():
    for n in (20, 7, 11):
        for j in range(n):
            assert orc.ratio(j, n) == nearest_f32_of_fraction(Fraction(j, n))
    assert orc.ratio(0, 20) == 0 and orc.ratio(19, 20) < 1


def test_pow_special_cases():
    for a in (F32(0), F32(1e-30), F32(0.5), F32(1), F32(37.25)):
        assert orc.cr_pow(a, F32(0)) == F32(1)
    for j in range(1, 20):
        r = orc.ratio(j, 20)
        assert orc.cr_pow(F32(1), r) == F32(1)
        assert orc.cr_pow(F32(0), r) == F32(0)
    assert orc.cr_pow(F32(256), F32(0.25)) == F32(4)
    assert orc.cr_pow(F32(256), F32(0.75)) == F32(64)
    assert orc.cr_pow(F32(2.0 ** -20), F32(0.5)) == F32(2.0 ** -10)
    assert orc.cr_pow(F32(2.0 ** 40), F32(0.75)) == F32(2.0 ** 30)


@pytest.mark.parametrize("p", [1, 2, 3])
def test_pow_quarter_exponents_by_exact_integer_powers(p):
    """r = p/4 is exact in fp32: y is the correctly rounded a^(p/4) iff lo^4 < a^p < hi^4 for the
    midpoints lo, hi around y (exact rational arithmetic, no transcendental function)."""
    rng = np.random.default_rng(10 + p)
    a_vals = np.concatenate([rng.random(150) * 50, rng.random(50) * 1e-3]).astype(F32)
    r = F32(p / 4)
    for a in a_vals:
        if a == 0:
            continue
        y = orc.cr_pow(a, r)
        lo, hi = midpoints(y)
        ap = Fraction(float(a)) ** p
        assert lo ** 4 < ap < hi ** 4, (a, p, y)


def _mp_round_to_f32(y) -> np.float32:
    f = F32(float(y))
    best = None
    for c in (np.nextafter(f, F32(-np.inf)), f, np.nextafter(f, F32(np.inf))):
        d = abs(mpmath.mpf(float(c)) - y)
        if best is None or d < best[0]:
            best = (d, c)
    return F32(best[1])


def test_pow_matches_mpmath_200_bits_random():
    rng = np.random.default_rng(21)
    a_vals = np.concatenate([rng.random(60) * 40, 10.0 ** rng.uniform(-8, 3, 60)]).astype(F32)
    with mpmath.workprec(200):
        for i, a in enumerate(a_vals):
            j = 1 + i % 19
            r = orc.ratio(j, 20)
            ref = _mp_round_to_f32(mpmath.power(mpmath.mpf(float(a)), mpmath.mpf(float(r))))
            assert orc.cr_pow(a, r) == ref, (a, r)


def near_midpoint_cases(count=12, seed=5, rel=2.0 ** -34):
    """(a, j) pairs whose real power a^(j/20) lies within ``rel`` (relative) of a float32 midpoint,
    screened with fp64 pow and confirmed with mpmath at 200 bits."""
    rng = np.random.default_rng(seed)
    found = []
    with mpmath.workprec(200):
        while len(found) < count:
            a = (rng.random(200000) * 30 + 1e-3).astype(F32)
            j = rng.integers(1, 20, a.shape[0])
            r = (j.astype(F32) / F32(20)).astype(F32)
            y = np.power(a.astype(np.float64), r.astype(np.float64))
            bits = y.view(np.uint64) & np.uint64((1 << 29) - 1)
            cand = np.nonzero(np.abs(bits.astype(np.int64) - (1 << 28)) < (1 << 14))[0]
            for i in cand:
                ym = mpmath.power(mpmath.mpf(float(a[i])), mpmath.mpf(float(r[i])))
                f = F32(float(ym))
                lo, hi = midpoints(f)
                dist = min(abs(mpmath.mpf(lo.numerator) / lo.denominator - ym),
                           abs(mpmath.mpf(hi.numerator) / hi.denominator - ym)) / ym
                if dist < rel:
                    found.append((F32(a[i]), int(j[i])))
                if len(found) >= count:
                    break
    return found


def test_pow_near_fp32_midpoints_matches_mpmath():
    cases = near_midpoint_cases()
    assert len(cases) >= 12
    with mpmath.workprec(200):
        for a, j in cases:
            r = orc.ratio(j, 20)
            ref = _mp_round_to_f32(mpmath.power(mpmath.mpf(float(a)), mpmath.mpf(float(r))))
            assert orc.cr_pow(a, r) == ref, (a, j)


def test_scale_table_closed_form_two_channels():
    """act = [1, 4] at ratio 1/2: t = [1, 2], d = nearest fp32 of sqrt(2), s = nearest fp32 of t / d."""
    s = orc.scale_candidates(np.array([1.0, 4.0], F32), F32(0.5))
    with localcontext() as ctx:
        ctx.prec = 80
        d = nearest_f32_of_fraction(Fraction(Decimal(2).sqrt()))
    assert s[0] == nearest_f32_of_fraction(Fraction(1) / Fraction(float(d)))
    assert s[1] == nearest_f32_of_fraction(Fraction(2) / Fraction(float(d)))


def test_scale_table_invariants():
    rng = np.random.default_rng(7)
    act = np.concatenate([rng.random(250).astype(F32) * 2, np.array([0.0, 1e-9, 35.0], F32)])
    act = act.astype(F32)
    T = orc.scale_table(act, 20)
    assert T.shape == (20, act.shape[0]) and T.dtype == F32
    assert np.all(T[0] == F32(1.0)), "ratio 0 must give scales of exactly one"
    order = np.argsort(act, kind="stable")
    for j in range(1, 20):
        s = T[j]
        prod = float(s.max()) * float(s.min())
        assert abs(prod - 1.0) <= 4 * 2.0 ** -23, (j, prod)
        assert np.all(np.diff(s[order]) >= 0), "scales must follow the order of the statistic"
        # a zero statistic hits the 1e-4 floor; 1e-9 ** r does too once r > 4/9
        assert s[-3] == s.min()
        if j >= 9:
            assert s[-2] == s[-3]
        else:
            assert s[-2] > s[-3]
        assert s[-1] == s.max()


# ------------------------------------------------------------------------------------------------ a3
def test_quantizer_codes_and_error_bound_random_groups():
    rng = np.random.default_rng(11)
    wp = (rng.standard_normal((64, 512)) * rng.uniform(0.001, 3, (64, 1))).astype(F32)
    wp[:8] += F32(5)              # all-positive groups: negative zero points
    wp[8:12] -= F32(7)            # all-negative groups: zero points above 15
    q, step, z, deq = orc.quantize_groups(wp)
    assert np.all(q == np.rint(q)) and q.min() >= 0 and q.max() <= 15
    assert np.all(z == np.rint(z))
    assert (z[:8] < 0).any() and (z[8:12] > 15).any()
    raw = np.rint(wp.reshape(64, 4, 128) / step[..., None]) + z[..., None]
    unclipped = ((raw >= 0) & (raw <= 15)).reshape(64, 512)
    err = np.abs(wp.astype(np.float64) - deq.astype(np.float64))
    bound = np.repeat(step.astype(np.float64), 128, axis=1) / 2 * (1 + 2.0 ** -22)
    assert np.all(err[unclipped] <= bound[unclipped])


def test_quantizer_brute_force_over_all_16_levels():
    """Given (step, z), each code is the level nearest to w' among all 16, by exact arithmetic;
    a near-tie (exact quotient within 2 ulp of a half-integer) may go either way."""
    rng = np.random.default_rng(12)
    wp = (rng.standard_normal((24, 256)) * rng.uniform(0.01, 2, (24, 1))).astype(F32)
    q, step, z, _ = orc.quantize_groups(wp)
    for o in range(wp.shape[0]):
        for g in range(2):
            st = Fraction(float(step[o, g]))
            zz = Fraction(float(z[o, g]))
            for kk in range(128):
                w = Fraction(float(wp[o, g * 128 + kk]))
                dists = [abs(w - (lvl - zz) * st) for lvl in range(16)]
                best = min(dists)
                chosen = int(q[o, g * 128 + kk])
                if dists[chosen] != best:
                    quo = w / st
                    half = Fraction(int(np.floor(float(quo)))) + Fraction(1, 2)
                    assert abs(quo - half) <= 2 * abs(quo) * Fraction(1, 2 ** 23), (o, g, kk)


def test_quantizer_step_and_zero_rounding_is_exact_division():
    rng = np.random.default_rng(13)
    wp = (rng.standard_normal((16, 384)) * 0.05).astype(F32)
    q, step, z, _ = orc.quantize_groups(wp)
    g = wp.reshape(16, 3, 128)
    for o in range(16):
        for gi in range(3):
            mx, mn = g[o, gi].max(), g[o, gi].min()
            rng_f = nearest_f32_of_fraction(Fraction(float(mx)) - Fraction(float(mn)))
            st = nearest_f32_of_fraction(Fraction(float(rng_f)) / 15)
            st = max(st, F32(1e-5))
            assert step[o, gi] == st
            zq = nearest_f32_of_fraction(-Fraction(float(mn)) / Fraction(float(st)))
            assert z[o, gi] == F32(np.rint(zq)) + F32(0)


def test_quantizer_constant_groups_use_step_floor():
    wp = np.zeros((3, 256), F32)
    wp[0, :128] = F32(0.3)
    wp[1, :] = F32(-2.5)
    q, step, z, deq = orc.quantize_groups(wp)
    assert np.all(step == F32(1e-5))
    assert np.all(q == 0)
    assert np.all(np.abs(deq.astype(np.float64) - wp) <= 0.5e-5 * (1 + 1e-6))
    assert not np.signbit(z).any() or np.all(z[np.signbit(z)] != 0), "zero points must not be -0"
    assert np.all(np.signbit(z[2]) == False)  # noqa: E712


def test_quantizer_noise_rms_is_step_over_sqrt12():
    """Uniform rounding noise has standard deviation step/sqrt(12) (section 2.1 of the hncyxsy.com outlier
    page); checked within 5% on groups whose values are spread over many levels."""
    rng = np.random.default_rng(14)
    wp = rng.uniform(-1, 1, (512, 1024)).astype(F32)
    q, step, z, deq = orc.quantize_groups(wp)
    err = (wp.astype(np.float64) - deq).reshape(512, 8, 128) / step[..., None].astype(np.float64)
    rms = np.sqrt(np.mean(err ** 2))
    assert abs(rms - 1 / np.sqrt(12)) < 0.05 / np.sqrt(12)


def on_grid_weight(O, K, seed):
    """W = (q - z) * 2^-7 with levels 0 and 15 present in every group and z in [0, 15] per group."""
    rng = np.random.default_rng(seed)
    q = rng.integers(0, 16, (O, K))
    q[:, 0::128] = 0
    q[:, 1::128] = 15
    z = np.repeat(rng.integers(0, 16, (O, K // 128)), 128, axis=1)
    return inputs.f32_to_bf16_bits(((q - z) * 2.0 ** -7).astype(F32))


def test_on_grid_weight_gives_zero_loss_at_ratio_zero():
    W = on_grid_weight(96, 256, 15)
    X = inputs.random_bf16((200, 256), 16, outliers=3, factor=40)
    res = orc.search(X, W, n_grid=20)
    assert res["losses"][0] == 0.0
    assert res["best_j"] == 0
    w_hat, _, _, _ = orc.pseudo_quantize(W, np.ones(256, F32))
    assert np.array_equal(w_hat, inputs.bf16_bits_to_f32(W))


def torch_plain_rtn(w_f32: np.ndarray) -> np.ndarray:
    """Independent plain round-to-nearest INT4 (no scaling), written with torch float32 ops."""
    w = torch.from_numpy(w_f32.copy()).reshape(-1, 128)
    hi = w.amax(dim=1, keepdim=True)
    lo = w.amin(dim=1, keepdim=True)
    st = torch.clamp((hi - lo) / 15.0, min=float(np.float32(1e-5)))
    zp = torch.round(-lo / st)
    q = torch.clamp(torch.round(w / st) + zp, 0, 15)
    return ((q - zp) * st).reshape(w_f32.shape).numpy()


def test_ratio_zero_equals_plain_rtn():
    wl = inputs.workload(1)
    X, W, _ = inputs.make_inputs(wl)
    res = orc.search(X, W, n_grid=20)
    rtn = torch_plain_rtn(inputs.bf16_bits_to_f32(W))
    assert res["losses"][0] == orc.loss_of(X, W, rtn)
    w_hat, _, _, _ = orc.pseudo_quantize(W, res["table"][0])
    assert np.array_equal(w_hat, rtn)


def test_awq_beats_rtn_with_outlier_channels():
    """The pages' claim (gsyq.cn AWQ page, section 三): scaling protects outlier channels, so some
    ratio beats plain RTN on activations with outliers."""
    X, W, _ = inputs.make_inputs(inputs.workload(1))
    res = orc.search(X, W, n_grid=20)
    assert res["best_j"] > 0
    assert res["losses"][res["best_j"]] < 0.9 * res["losses"][0]


# ------------------------------------------------------------------------------------------------ a4
def test_scaling_identity_without_quantization():
    """X W^T == (X diag(s)^-1)(diag(s) W)^T (section 一 of the gsyq.cn AWQ page), in fp64."""
    X = inputs.random_bf16((96, 256), 31, outliers=2, factor=30)
    W = inputs.random_bf16((80, 256), 32, scale=0.02)
    act = orc.act_mean(X)
    s = orc.scale_candidates(act, orc.ratio(13, 20)).astype(np.float64)
    x = inputs.bf16_bits_to_f32(X).astype(np.float64)
    w = inputs.bf16_bits_to_f32(W).astype(np.float64)
    ref = x @ w.T
    alt = (x / s[None, :]) @ (w * s[None, :]).T
    assert np.max(np.abs(ref - alt)) <= 1e-12 * np.max(np.abs(ref))
    # with an identity quantizer the oracle's scale/unscale round trip leaves only fp32 rounding
    w_hat = ((inputs.bf16_bits_to_f32(W) * s.astype(F32)[None, :]).astype(F32) / s.astype(F32)[None, :])
    assert np.max(np.abs(w_hat - inputs.bf16_bits_to_f32(W))) <= 2.0 ** -23 * np.abs(w).max()
    assert orc.loss_of(X, W, w_hat) < 1e-10 * orc.loss_of(X, W, np.zeros_like(w_hat))


def test_loss_delta_form_equals_two_gemm_form():
    X = inputs.random_bf16((384, 256), 41, outliers=3, factor=50)
    W = inputs.random_bf16((192, 256), 42, scale=0.02)
    s = orc.scale_candidates(orc.act_mean(X), orc.ratio(9, 20))
    w_hat, _, _, _ = orc.pseudo_quantize(W, s)
    x = inputs.bf16_bits_to_f32(X).astype(np.float64)
    w = inputs.bf16_bits_to_f32(W).astype(np.float64)
    two = np.mean((x @ w.T - x @ w_hat.astype(np.float64).T) ** 2)
    assert abs(orc.loss_of(X, W, w_hat) - two) <= 1e-12 * two


def test_loss_hand_example_mean_normalisation():
    """One off-grid weight, a unit activation on its channel: the loss is err^2 / (N * O)."""
    W = on_grid_weight(2, 128, 51).astype(np.uint16)
    wf = inputs.bf16_bits_to_f32(W).copy()
    k = 5
    wf[1, k] = wf[1, k] + F32(2.0 ** -9)         # a quarter step off the grid, min/max unchanged
    assert wf[1, k] < wf[1].max() and wf[1, k] > wf[1].min()
    W2 = inputs.f32_to_bf16_bits(wf)
    x = np.zeros((3, 128), F32)
    x[0, k] = 1.0
    X = inputs.f32_to_bf16_bits(x)
    w_hat, _, _, _ = orc.pseudo_quantize(W2, np.ones(128, F32))
    assert orc.loss_of(X, W2, w_hat) == (2.0 ** -9) ** 2 / (3 * 2)


# ------------------------------------------------------------------------------------------------ a5
def test_argmin_first_minimum_wins():
    assert orc.argmin_first([3.0, 1.0, 1.0, 2.0]) == 1
    assert orc.argmin_first([1.0, 1.0]) == 0
    assert orc.argmin_first([5.0, 4.0, 3.0, 3.0, 3.0]) == 2
    assert orc.argmin_first([0.5]) == 0
    assert orc.argmin_first([2.0, 1.0, 0.25, 0.25 + 1e-18, 0.25]) == 2


# ------------------------------------------------------------------------------------------------ a6
def test_pack_layout_and_round_trip():
    q = np.zeros((2, 16), np.uint8)
    q[0, :8] = np.arange(8)
    q[1, 8] = 15
    words = orc.pack_codes(q)
    assert words[0, 0] == 0x76543210 and words[0, 1] == 0
    assert words[1, 0] == 0 and words[1, 1] == 0x0000000F
    rng = np.random.default_rng(61)
    q = rng.integers(0, 16, (33, 256)).astype(np.uint8)
    assert np.array_equal(orc.unpack_codes(orc.pack_codes(q), 256), q)


def test_shared_input_concatenation_is_one_search():
    """Several linears on one input share one scale (NormLinearSubgraph on the msModelSlim AWQ page):
    the loss of the stacked weight is the row-weighted mean of the per-linear losses."""
    X = inputs.random_bf16((160, 256), 71, outliers=2, factor=60)
    Wq = inputs.random_bf16((128, 256), 72, scale=0.02)
    Wk = inputs.random_bf16((64, 256), 73, scale=0.02)
    W = np.concatenate([Wq, Wk])
    act = orc.act_mean(X)
    T = orc.scale_table(act, 20)
    res = orc.search(X, W, n_grid=20, act=act, table=T)
    for j in (0, 7, 19):
        lq = orc.loss_of(X, Wq, orc.pseudo_quantize(Wq, T[j])[0])
        lk = orc.loss_of(X, Wk, orc.pseudo_quantize(Wk, T[j])[0])
        assert abs(res["losses"][j] - (128 * lq + 64 * lk) / 192) <= 1e-12 * res["losses"][j]


# ------------------------------------------------------------------------------------------ folding
def test_bf16_rounding_is_nearest_even():
    rng = np.random.default_rng(91)
    x = (rng.standard_normal(4000) * 10.0 ** rng.uniform(-6, 6, 4000)).astype(F32)
    got = inputs.bf16_bits_to_f32(orc.round_f32_to_bf16(x))
    for v, g in zip(x[:500], got[:500]):
        lo = np.float32(inputs.bf16_bits_to_f32(np.array([orc.round_f32_to_bf16(np.array([v]))[0]]))[0])
        assert g == lo
        # exact check: no bf16 value is strictly closer
        up = inputs.bf16_bits_to_f32((orc.round_f32_to_bf16(np.array([v])).astype(np.uint32) + 1).astype(np.uint16))[0]
        dn = inputs.bf16_bits_to_f32((orc.round_f32_to_bf16(np.array([v])).astype(np.int64) - 1).astype(np.uint16))[0]
        d = abs(Fraction(float(g)) - Fraction(float(v)))
        assert d <= abs(Fraction(float(up)) - Fraction(float(v))) and d <= abs(Fraction(float(dn)) - Fraction(float(v)))
    # ties go to the even pattern: 1 + 2^-8 lies halfway between 1 and 1 + 2^-7
    assert orc.round_f32_to_bf16(np.array([1 + 2.0 ** -8], F32))[0] == 0x3F80
    assert orc.round_f32_to_bf16(np.array([1 + 3 * 2.0 ** -8], F32))[0] == 0x3F82


def test_fold_identity_and_powers_of_two():
    A = inputs.random_bf16((7, 64), 92, scale=0.5)
    one = np.ones(64, F32)
    assert np.array_equal(orc.fold_columns(A, one, False), A)
    assert np.array_equal(orc.fold_rows(A, np.ones(7, F32), True), A)
    two = np.full(64, 4.0, F32)
    assert np.array_equal(inputs.bf16_bits_to_f32(orc.fold_columns(A, two, False)), inputs.bf16_bits_to_f32(A) * 4)
    assert np.array_equal(inputs.bf16_bits_to_f32(orc.fold_columns(A, two, True)), inputs.bf16_bits_to_f32(A) / 4)


def test_folded_norm_linear_keeps_the_output():
    """gamma / s on the norm and W diag(s) on the linear give the same output (section 一 of the gsyq.cn
    AWQ page), up to the bf16 rounding of the folded parameters."""
    rng = np.random.default_rng(93)
    K, O = 256, 64
    xn = inputs.random_bf16((32, K), 94)                       # normalised activations before gamma
    gamma = inputs.f32_to_bf16_bits((1 + 0.1 * rng.standard_normal(K)).astype(F32))
    W = inputs.random_bf16((O, K), 95, scale=0.02)
    act = orc.act_mean(inputs.random_bf16((200, K), 96, outliers=3, factor=50))
    s = orc.scale_candidates(act, orc.ratio(11, 20))
    g2 = orc.fold_columns(gamma[None, :], s, True)[0]
    W2 = orc.fold_columns(W, s, False)
    f = lambda b: inputs.bf16_bits_to_f32(b).astype(np.float64)  # noqa: E731
    ref = (f(xn) * f(gamma)[None, :]) @ f(W).T
    alt = (f(xn) * f(g2)[None, :]) @ f(W2).T
    mag = np.abs(f(xn) * f(gamma)[None, :]) @ np.abs(f(W)).T
    assert np.all(np.abs(alt - ref) <= 2 * 2.0 ** -8 * mag)


def test_folded_linear_linear_keeps_the_output():
    """Rows (and bias) of linear1 divided by s, columns of linear2 multiplied by s."""
    K, H, O = 128, 256, 96
    x = inputs.random_bf16((16, K), 97)
    W1 = inputs.random_bf16((H, K), 98, scale=0.05)
    b1 = inputs.random_bf16((1, H), 99, scale=0.1)[0]
    W2 = inputs.random_bf16((O, H), 100, scale=0.05)
    act = orc.act_mean(inputs.random_bf16((64, H), 101, outliers=2, factor=30))
    s = orc.scale_candidates(act, orc.ratio(15, 20))
    f = lambda b: inputs.bf16_bits_to_f32(b).astype(np.float64)  # noqa: E731
    h = f(x) @ f(W1).T + f(b1)[None, :]
    ref = h @ f(W2).T
    h2 = f(x) @ f(orc.fold_rows(W1, s, True)).T + f(orc.fold_columns(b1[None, :], s, True)[0])[None, :]
    alt = h2 @ f(orc.fold_columns(W2, s, False)).T
    mag = np.abs(h) @ np.abs(f(W2)).T
    assert np.all(np.abs(alt - ref) <= 3 * 2.0 ** -8 * mag + 1e-12)


# ------------------------------------------------------------------------------------------ W4A16
def test_dequant_from_packed_codes_equals_the_quantizers_dequant():
    W = inputs.random_bf16((48, 384), 111, scale=0.03)
    s = orc.scale_candidates(orc.act_mean(inputs.random_bf16((64, 384), 112, outliers=2, factor=40)),
                             orc.ratio(9, 20))
    wp = (inputs.bf16_bits_to_f32(W) * s[None, :]).astype(F32)
    _, _, _, deq = orc.quantize_groups(wp)
    words, steps, zeros = orc.quantize_pack(W, s)
    assert np.array_equal(orc.dequant_w4(words, steps, zeros), deq)


def test_w4a16_hand_examples():
    O, K = 8, 128
    q = np.full((O, K), 8, np.uint8)
    words = orc.pack_codes(q)
    zeros = np.full((O, 1), 8.0, F32)
    steps = np.full((O, 1), 0.25, F32)
    x = inputs.random_bf16((3, K), 113)
    assert np.all(orc.w4a16_matmul(x, words, steps, zeros) == 0.0)
    rng = np.random.default_rng(114)
    q = rng.integers(0, 16, (O, K)).astype(np.uint8)
    y = orc.w4a16_matmul(x, orc.pack_codes(q), np.ones((O, 1), F32), np.zeros((O, 1), F32))
    assert np.array_equal(y, inputs.bf16_bits_to_f32(x).astype(np.float64) @ q.T.astype(np.float64))
    for weights in ("bf16", "fp32"):
        y = orc.w4a16_matmul(x, orc.pack_codes(q), np.ones((O, 1), F32), np.zeros((O, 1), F32), weights=weights)
        assert np.array_equal(y, inputs.bf16_bits_to_f32(x).astype(np.float64) @ q.T.astype(np.float64))


def test_w4a16_fp32_weights_one_hot_columns():
    """With X' one-hot at in-feature k (value 1), row m of the fp32-weight product is column k of the
    dequantized weight exactly, q - z times step rounded once; the bf16-weight product is its bf16 rounding."""
    O, K = 16, 256
    rng = np.random.default_rng(115)
    q = rng.integers(0, 16, (O, K)).astype(np.uint8)
    steps = (rng.random((O, K // 128)) * 0.01 + 1e-3).astype(F32)
    zeros = rng.integers(-3, 19, (O, K // 128)).astype(F32)
    ks = np.array([0, 1, 4, 7, 8, 127, 128, 200, 255])
    x = np.zeros((ks.size, K), np.uint16)
    x[np.arange(ks.size), ks] = 0x3F80  # bf16 1.0
    words = orc.pack_codes(q)
    y32 = orc.w4a16_matmul(x, words, steps, zeros, weights="fp32")
    y16 = orc.w4a16_matmul(x, words, steps, zeros, weights="bf16")
    for i, k in enumerate(ks):
        g = k // 128
        want = np.array([np.float32(np.float32(float(q[o, k]) - zeros[o, g]) * steps[o, g]) for o in range(O)])
        assert np.array_equal(y32[i], want.astype(np.float64))
        assert np.array_equal(y16[i], inputs.bf16_bits_to_f32(orc.round_f32_to_bf16(want)).astype(np.float64))


# ------------------------------------------------------------------------------------------ scale rules
def test_closed_grid_points():
    assert [orc.closed_grid(j, 11) for j in (0, 10)] == [0.0, 1.0]
    for j in range(11):
        assert orc.closed_grid(j, 11) == nearest_f32_of_fraction(Fraction(j, 10))
    assert orc.closed_grid(0, 1) == 0.0


def test_weight_aware_rule_end_points():
    """p = 1 leaves act / (1 + 1e-6) (wmean^0 = 1); p = 0 leaves 1 / (wmean + 1e-6); both normalised."""
    rng = np.random.default_rng(121)
    act = (rng.random(200) * 3 + 0.01).astype(F32)
    wm = (rng.random(200) * 0.05 + 0.001).astype(F32)
    T = orc.scale_table_weight_aware(act, wm, 5)
    for row, expect_order in ((T[-1], act), (T[0], -wm)):
        order = np.argsort(expect_order, kind="stable")
        assert np.all(np.diff(row[order]) >= 0)
        assert abs(float(row.max()) * float(row.min()) - 1) <= 4 * 2.0 ** -23
    eps = Fraction(float(F32(1e-6)))
    one_plus = nearest_f32_of_fraction(1 + eps)
    t = [nearest_f32_of_fraction(Fraction(float(a)) / Fraction(float(one_plus))) for a in act]
    t = np.maximum(np.array(t, F32), F32(1e-4))
    d = np.sqrt(F32(t.max() * t.min()))
    assert np.array_equal(T[-1], (t / d).astype(F32))


def test_rms_rule_end_points_and_sum():
    rng = np.random.default_rng(122)
    act = np.concatenate([rng.random(300) * 4, [0.0, 1e-7]]).astype(F32)
    T = orc.scale_table_rms(act, 11)
    assert np.all(T[0] == F32(1.0)), "alpha = 0 must give scales of exactly one"
    a = np.maximum(act, F32(1e-5))
    rms = np.sqrt(np.mean(T[-1].astype(np.float64) ** 2))
    assert abs(rms - 1) < 1e-5
    order = np.argsort(a, kind="stable")
    for j in range(11):
        assert np.all(np.diff(T[j][order]) >= 0)
    # the fixed-order fp64 sum of the fp32 squares is within one fp64 rounding per chunk of the exact sum
    sq = (a * a).astype(F32)
    exact = sum(Fraction(float(v)) for v in sq)
    assert abs(Fraction(float(orc._sum_sq_fixed(a))) - exact) <= exact * Fraction(1, 2 ** 45)


def test_search_rules_pick_a_ratio_that_beats_rtn():
    X, W, _ = inputs.make_inputs(inputs.workload(1))
    for mode in ("weight_aware", "rms"):
        res = orc.search(X, W, n_grid=11 if mode == "rms" else 20, mode=mode)
        assert res["losses"][res["best_j"]] <= res["losses"][0]


# ------------------------------------------------------------------------------------------------ f4
def test_int8_worked_example_of_the_outlier_page():
    """The page's two cases: one outlier of 23 wipes 0.03 out (code 0); without it 0.03 keeps code 38."""
    import json
    import os
    with open(os.path.join(os.path.dirname(__file__), "golden", "int8_outlier_example.json")) as f:
        cases = json.load(f)["cases"]
    for c in cases:
        wp = np.array([[c["max_abs"], c["x"], -c["max_abs"] / 4, 0.0]], F32)
        q, step, deq = orc.quantize_rows_int8(wp)
        assert round(float(step[0]), c["scale_digits"]) == c["scale_printed"]
        assert int(q[0, 1]) == c["code"]
        assert q[0, 0] == 127
        if "dequant_printed" in c:
            assert round(float(deq[0, 1]), c["dequant_digits"]) == c["dequant_printed"]
            assert abs(float(deq[0, 1]) - c["x"]) / c["x"] < c["relative_error_below"]
        else:
            assert float(deq[0, 1]) == c["dequant"]


def test_int8_step_is_exact_division_and_codes_nearest_of_255_levels():
    """step = nearest fp32 of max|w'| / 127; each code is the nearest of the 255 levels by exact arithmetic
    (a near-tie may go either way); the row's max |w'| gets code +-127."""
    rng = np.random.default_rng(131)
    wp = (rng.standard_normal((12, 96)) * rng.uniform(0.001, 4, (12, 1))).astype(F32)
    q, step, deq = orc.quantize_rows_int8(wp)
    for o in range(wp.shape[0]):
        amax = max(abs(Fraction(float(v))) for v in wp[o])
        assert step[o] == max(nearest_f32_of_fraction(amax / 127), F32(1e-5))
        st = Fraction(float(step[o]))
        for k in range(wp.shape[1]):
            w = Fraction(float(wp[o, k]))
            quo = w / st
            nearest = min(range(-127, 128), key=lambda lvl: abs(quo - lvl))
            if int(q[o, k]) != nearest:
                half = Fraction(int(np.floor(float(quo)))) + Fraction(1, 2)
                assert abs(quo - half) <= 2 * abs(quo) * Fraction(1, 2 ** 23), (o, k)
            assert deq[o, k] == nearest_f32_of_fraction(Fraction(int(q[o, k])) * st)
        kmax = int(np.argmax(np.abs(wp[o])))
        assert abs(int(q[o, kmax])) == 127 and np.sign(q[o, kmax]) == np.sign(wp[o, kmax])


def test_int8_symmetry_zero_rows_and_error_bound():
    rng = np.random.default_rng(132)
    wp = (rng.standard_normal((8, 256)) * 0.3).astype(F32)
    wp[3] = 0.0
    q, step, deq = orc.quantize_rows_int8(wp)
    qn, stepn, _ = orc.quantize_rows_int8(-wp)
    assert np.array_equal(step, stepn) and np.array_equal(q, -qn), "the quantizer is odd-symmetric"
    assert step[3] == F32(1e-5) and np.all(q[3] == 0)
    assert q.min() >= -127 and q.max() <= 127
    err = np.abs(wp.astype(np.float64) - deq.astype(np.float64))
    assert np.all(err <= step[:, None].astype(np.float64) / 2 * (1 + 2.0 ** -21) + 1e-30)


def test_int8_search_ratio_zero_is_per_channel_rtn_and_beats_int4():
    X, W, _ = inputs.make_inputs(inputs.workload(1))
    res8 = orc.search(X, W, n_grid=20, quant="int8")
    res4 = orc.search(X, W, n_grid=20)
    w = inputs.bf16_bits_to_f32(W)
    q, step, deq = orc.quantize_rows_int8(w)  # s = 1 at ratio 0 (act^0 = 1, normalised to 1)
    assert np.all(res8["table"][0] == F32(1))
    assert res8["losses"][0] == orc.loss_of(X, W, deq)
    assert res8["codes"].dtype == np.int8 and res8["zeros"] is None
    assert res8["losses"][res8["best_j"]] <= res8["losses"][0]
    # 255 levels per channel against 16 per group of 128: far smaller error on these Gaussian rows
    assert res8["losses"].min() < res4["losses"].min() / 10
