"""Pins of the data-free UOS objective (oracle/uos_theory.py): hand-computed
values of E, the closed forms of Delta on both branches, and the argmin of J
under several wrapped block-maximum densities (Fig. 2)."""
import numpy as np
import pytest

from conftest import golden
from oracle import uos_theory as T

G = golden("uos_objective.json")


def test_projection_is_nearest_grid_point():
    for v in np.linspace(0, 9, 901):
        p = T.projection(v)
        assert p in T.GRID
        if v < 6:
            assert all(abs(v - p) <= abs(v - g) + 1e-15 for g in T.GRID)
        else:
            assert p == 6.0


@pytest.mark.parametrize("x", ["3", "4", "6"])
def test_E_hand_values(x):
    assert T.E(float(x)) == pytest.approx(G["E_values_hand_computed"][x], abs=1e-15)


def test_E_matches_numerical_integration():
    from scipy.integrate import quad
    for x in (0.3, 1.1, 2.7, 3.9, 5.5, 7.25, 8.0):
        pts = [p for p in T._BP if p < x]
        num, _ = quad(lambda v: (v - T.projection(v)) ** 2, 0, x, points=pts, limit=200)
        assert T.E(x) == pytest.approx(num, rel=1e-9, abs=1e-12)


def test_delta_first_branch_constant_negative():
    lo, hi = G["delta_first_branch"]["q_range"]
    for q in np.linspace(lo, hi, 41):
        assert T.Delta(q) == pytest.approx(G["delta_first_branch"]["value"], abs=1e-12)


def test_delta_second_branch_factors():
    lo, hi = G["delta_second_branch"]["q_range"]
    for q in np.linspace(lo, hi, 41):
        assert T.Delta(q) == pytest.approx((4 * q - 29) * (4 * q - 27) / 8, abs=1e-12)
    assert T.root_of_Delta() == pytest.approx(G["delta_second_branch"]["root"], abs=1e-12)


@pytest.mark.parametrize("name", list(T.DENSITIES))
def test_argmin_J_is_29_over_4(name):
    q = T.argmin_J(T.DENSITIES[name])
    assert abs(q - G["q_star"]) < 1e-6, q


def test_J_ordering_of_the_three_rules():
    """The UOS boundary beats Qmax=6, OCP's effective boundary 8 and q=7 (OAS)."""
    for w in T.DENSITIES.values():
        j = {q: T.J(q, w) for q in (6.0, 7.0, 7.25, 8.0)}
        assert j[7.25] < j[7.0] < j[6.0]
        assert j[7.25] < j[8.0]
