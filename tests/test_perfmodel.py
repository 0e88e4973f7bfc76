"""The linear time model's fit (FinDEP review, section "核心公式": t_e(m_e) = a + b*m_e)."""
import numpy as np
import pytest

from expert_ffn_layer_moe_b200.perfmodel import fit_linear, fit_multilinear


def test_exact_line():
    a, b, r2 = fit_linear([0, 1, 2], [1, 3, 5])
    assert (round(a, 12), round(b, 12), round(r2, 12)) == (1.0, 2.0, 1.0)


def test_no_linear_trend_has_zero_r2():
    # (0,0), (1,1), (2,0): best line is flat at 1/3, explaining none of the variance
    a, b, r2 = fit_linear([0, 1, 2], [0, 1, 0])
    assert abs(a - 1 / 3) < 1e-12 and abs(b) < 1e-12 and abs(r2) < 1e-12


def test_matches_polyfit_on_noisy_data():
    g = np.random.default_rng(0)
    m = np.array([0.06, 1, 4, 8, 16, 32, 64, 128, 256, 512])
    t = 0.05 + 0.0008 * m + g.normal(0, 0.003, m.size)
    a, b, r2 = fit_linear(m, t)
    pb, pa = np.polyfit(m, t, 1)
    assert np.allclose([a, b], [pa, pb], rtol=1e-10, atol=1e-12)
    assert np.isclose(r2, np.corrcoef(m, t)[0, 1] ** 2, rtol=1e-10)


def test_needs_two_points():
    with pytest.raises(ValueError):
        fit_linear([1], [1])


def test_multilinear_recovers_two_coefficients():
    touched = [8, 82, 128, 128, 128, 128]
    rows = [0.06, 1, 4, 16, 64, 256]
    t = [0.01 + 0.002 * a + 0.0005 * b for a, b in zip(touched, rows)]
    coef, r2 = fit_multilinear([touched, rows], t)
    assert np.allclose(coef, [0.01, 0.002, 0.0005]) and np.isclose(r2, 1.0)
