"""The oracle's float -> ternary quantizers (absmean, Lloyd; groups of 128) against facts that
do not come from the oracle: the closed-form Gaussian errors of both rules, numpy's binary16
rounding, exact cases and the descent property of Lloyd's algorithm.

"Scion: ternary MoE quantization with trained corrections", Findings: the deployable Lloyd
quantizer beats one-shot absmean; "Scion-35B-A3B" model card, Highlights: ternary Lloyd g128.
"""
import numpy as np
import pytest
from scipy.stats import norm

import oracle


def _dequant(codes, scales):
    return codes.astype(np.float64) * scales.view(np.float16).astype(np.float64)[:, None]


def _rel_err(w, codes, scales):
    return np.linalg.norm(w.astype(np.float64) - _dequant(codes, scales)) / np.linalg.norm(w.astype(np.float64))


def _gauss_closed_forms():
    """Relative RMS error of the two rules on N(0, 1) with the group statistics exact (infinite
    groups): absmean s = E|w| = sqrt(2/pi), threshold s/2; Lloyd's fixed point t = s/2,
    s = E[|w| | |w| > t] = pdf(t) / (1 - cdf(t))."""
    def mse(s, t):  # E[(w - s c)^2], c = sign(w) 1{|w| > t}
        return 1.0 - 2.0 * s * 2.0 * norm.pdf(t) + s * s * 2.0 * norm.sf(t)

    s_abs = np.sqrt(2.0 / np.pi)
    e_abs = np.sqrt(mse(s_abs, s_abs / 2))
    s = s_abs
    for _ in range(200):
        s = norm.pdf(s / 2) / norm.sf(s / 2)
    return e_abs, np.sqrt(mse(s, s / 2))


def test_closed_forms_match_the_lloyd_max_ternary_quantizer():
    e_abs, e_lloyd = _gauss_closed_forms()
    # the 3-level Lloyd-Max quantizer of a unit Gaussian has MSE 0.1902 (thresholds +-0.612)
    assert e_lloyd ** 2 == pytest.approx(0.1902, abs=2e-4)
    assert e_abs == pytest.approx(0.514, abs=1e-3)


@pytest.mark.parametrize("method,which", [(oracle.ABSMEAN, 0), (oracle.LLOYD, 1)])
def test_gaussian_relative_error(method, which):
    """Many Gaussian groups: the error approaches the closed form (groups of 128 estimate their
    statistics, which lowers it by a few thousandths)."""
    rng = np.random.default_rng(123)
    w = rng.standard_normal((8192, 128)).astype(np.float32)
    codes, scales = oracle.quantize(method, w)
    ref = _gauss_closed_forms()[which]
    err = _rel_err(w, codes, scales)
    assert ref - 0.006 <= err <= ref + 0.001, (err, ref)


def test_lloyd_never_worse_than_absmean_per_group():
    """Lloyd starts from the absmean codes and every step (centroid, nearest level) lowers the
    squared error, so no group may end worse (up to the fp16 rounding of the scale)."""
    rng = np.random.default_rng(5)
    w = np.concatenate([rng.standard_normal((512, 128)), rng.laplace(size=(512, 128)),
                        rng.standard_t(3, size=(512, 128))]).astype(np.float32)
    ca, sa = oracle.quantize(oracle.ABSMEAN, w)
    cl, sl = oracle.quantize(oracle.LLOYD, w)
    ea = ((w - _dequant(ca, sa)) ** 2).sum(1)
    el = ((w - _dequant(cl, sl)) ** 2).sum(1)
    assert (el <= ea * (1 + 2e-3) + 1e-12).all()
    assert el.sum() < 0.95 * ea.sum()


def test_lloyd_result_is_a_fixed_point():
    rng = np.random.default_rng(9)
    w = rng.standard_t(4, size=(256, 128)).astype(np.float32)
    codes, scales = oracle.quantize(oracle.LLOYD, w, iters=1000)
    a = np.abs(w.astype(np.float64))
    nz = codes != 0
    s = (a * nz).sum(1) / nz.sum(1)  # centroid of the final cells
    again = np.where(2 * a >= s[:, None], np.sign(w), 0).astype(np.int8)
    np.testing.assert_array_equal(again, codes)
    np.testing.assert_array_equal(scales, s.astype(np.float16).view(np.uint16))


def test_absmean_is_rounding_of_w_over_mean_abs():
    rng = np.random.default_rng(11)
    w = rng.standard_normal((256, 128)).astype(np.float32)
    codes, scales = oracle.quantize(oracle.ABSMEAN, w)
    s = np.abs(w.astype(np.float64)).mean(1)
    q = w / s[:, None]
    ref = np.clip(np.sign(q) * np.floor(np.abs(q) + 0.5), -1, 1).astype(np.int8)  # half away from zero
    np.testing.assert_array_equal(codes, ref)
    np.testing.assert_array_equal(scales, s.astype(np.float16).view(np.uint16))


def test_exact_groups():
    w = np.zeros((5, 128), np.float32)
    w[1] = 0.25                                                   # constant
    w[2] = np.where(np.arange(128) % 2, 3.0, -3.0)                # two levels +-a
    w[3, 17] = -2.0                                               # one nonzero weight
    w[4] = np.where(np.arange(128) % 3 == 0, 0.0, np.where(np.arange(128) % 3 == 1, 1.5, -1.5))
    for method in (oracle.ABSMEAN, oracle.LLOYD):
        codes, scales = oracle.quantize(method, w)
        assert (codes[0] == 0).all() and scales[0] == 0
        assert (codes[1] == 1).all() and np.float16(scales[1].view(np.float16)) == np.float16(0.25)
        np.testing.assert_array_equal(codes[2], np.sign(w[2]).astype(np.int8))
        assert scales[2].view(np.float16) == np.float16(3.0)
        if method == oracle.LLOYD:
            # exact reconstruction whenever the group already is ternary
            np.testing.assert_array_equal(_dequant(codes[3:], scales[3:]), w[3:])


def test_f16_rounding_matches_numpy():
    rng = np.random.default_rng(3)
    v = np.concatenate([rng.uniform(0, 1, 2000) * 10.0 ** rng.integers(-9, 5, 2000),
                        np.ldexp(np.arange(0, 1024, dtype=np.float64) + 0.5, -24),  # ties between subnormals
                        np.ldexp(2049.0 + 2 * np.arange(200), -11), [65504.0, 65519.9, 65520.0, 6e-8, 0.0]])
    got = np.array([oracle.f64_to_f16(x) for x in v], np.uint16)
    with np.errstate(over="ignore"):  # 65520 rounds to infinity
        ref = v.astype(np.float16).view(np.uint16)
    np.testing.assert_array_equal(got, ref)


def test_non_finite_weights_are_rejected():
    w = np.zeros((2, 128), np.float32)
    w[1, 5] = np.inf
    with pytest.raises(ValueError):
        oracle.quantize(oracle.ABSMEAN, w)
