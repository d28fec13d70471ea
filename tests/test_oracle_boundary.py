"""Pins of the near-tie classifier and of the walk information it reads.

The classifier decides which rows of a GPU/oracle comparison may legitimately hold a
different kept set (the walk of a row ends so close to tau, or two ranked masses are so
close, that float rounding of the masses can move the cut).  A classifier that is too
permissive would silently widen what "identical block sets" means, so every condition is
fed hand-built walk vectors just inside and just outside its 1e-5 band, and the walk
information that `oracle.select` reports is checked against walks worked out by hand.

Source of the rule: block sets must match exactly except where the cumulative-mass
boundary lies within 1e-5 of tau (the workload definition of the long-context sweep);
the selection itself follows the MapFlow page "MapFlow开源:大模型换班,Prefill为何能快20%?",
section "存不下、读得慢?三个工程优化手段", subsection 1 (blocks chosen by cumulative
attention probability).
"""
import numpy as np
import pytest

import oracle

EPS = oracle.BOUNDARY_EPS


def info(total, S, S_prev=-1.0, m_last=-1.0, m_next=-1.0):
    return np.array([total, S, S_prev, m_last, m_next], dtype=np.float64)


def test_eps_is_the_stated_band():
    assert EPS == 1e-5


def test_empty_row_is_boundary():
    assert oracle.is_boundary(info(0.0, 0.0), 0.9)


@pytest.mark.parametrize("side", [+1, -1])
def test_final_fraction_band(side):
    tau, total = 0.9, 1000.0
    # inside: |S/total - tau| = 0.9e-5 < 1e-5
    assert oracle.is_boundary(info(total, total * (tau + side * 0.9e-5)), tau)
    # outside: 1.1e-5
    assert not oracle.is_boundary(info(total, total * (tau + side * 1.1e-5)), tau)
    # far away
    assert not oracle.is_boundary(info(total, total * (tau + side * 1e-2)), tau)


@pytest.mark.parametrize("side", [+1, -1])
def test_prefinal_fraction_band(side):
    tau, total = 0.8, 4096.0
    S = total * 0.95  # the final fraction is far from tau
    assert oracle.is_boundary(info(total, S, total * (tau + side * 0.9e-5)), tau)
    assert not oracle.is_boundary(info(total, S, total * (tau + side * 1.1e-5)), tau)
    # S_prev < 0 means "no pre-final sum" (only the diagonal was kept): never flagged
    assert not oracle.is_boundary(info(total, S, -1.0), tau)


def test_close_masses_band():
    tau, total = 0.95, 1000.0
    S, S_prev = 990.0, 900.0  # both fractions far from tau
    band = EPS * total        # 0.01
    assert oracle.is_boundary(info(total, S, S_prev, 5.0, 5.0 - 0.9 * band), tau)
    assert not oracle.is_boundary(info(total, S, S_prev, 5.0, 5.0 - 1.1 * band), tau)
    # equal masses (an exact tie) are near ties too
    assert oracle.is_boundary(info(total, S, S_prev, 5.0, 5.0), tau)
    # missing last-kept or first-dropped mass (-1): never flagged by this condition
    assert not oracle.is_boundary(info(total, S, S_prev, -1.0, 5.0), tau)
    assert not oracle.is_boundary(info(total, S, S_prev, 5.0, -1.0), tau)
    # the band scales with the row total, not with the masses themselves
    assert not oracle.is_boundary(info(10 * total, 10 * S, 10 * S_prev, 5.0, 5.0 - 1.1 * 10 * band), tau)
    assert oracle.is_boundary(info(10 * total, 10 * S, 10 * S_prev, 5.0, 5.0 - 0.9 * 10 * band), tau)


def test_walk_info_hand_worked():
    # qb = 3, masses of key blocks 0..3; the diagonal (kb 3) is kept first, then the others by
    # (mass desc, kb asc): kb 1 (4.0), kb 2 (2.0), kb 0 (1.0).  total = 10.
    m = np.array([1.0, 4.0, 2.0, 3.0])
    # tau = 0.75: target 7.5; S = 3 -> 7 -> 9 stops after kb 2
    kept, inf = oracle.select(m, 3, 0.75)
    assert kept.tolist() == [1, 2, 3]
    assert inf.tolist() == [10.0, 9.0, 7.0, 2.0, 1.0]
    assert not oracle.is_boundary(inf, 0.75)
    # tau = 0.7: S reaches exactly 7 = tau * total after kb 1: on the boundary itself
    kept, inf = oracle.select(m, 3, 0.7)
    assert kept.tolist() == [1, 3]
    assert inf.tolist() == [10.0, 7.0, 3.0, 4.0, 2.0]
    assert oracle.is_boundary(inf, 0.7)
    # only the diagonal kept: no pre-final sum and no last-kept candidate
    kept, inf = oracle.select(m, 3, 0.2)
    assert kept.tolist() == [3]
    assert inf.tolist() == [10.0, 3.0, -1.0, -1.0, 4.0]
    assert not oracle.is_boundary(inf, 0.2)
    # every block kept: no first-dropped candidate
    kept, inf = oracle.select(m, 3, 1.0)
    assert kept.tolist() == [0, 1, 2, 3]
    assert inf[4] == -1.0
    assert oracle.is_boundary(inf, 1.0)  # at tau = 1 the walk ends on S / total = 1 by definition


def test_walk_landing_just_inside_and_outside_the_band():
    # masses built so the walk's final fraction lands 0.5e-5 (inside) or 2e-5 (outside) above tau
    tau = 0.9
    for off, flagged in ((0.5e-5, True), (2e-5, False)):
        # diag 0.5, then a 0.4 + off block ends the walk at 0.9 + off of a total of 1
        m = np.array([0.1 - off, 0.4 + off, 0.5])
        kept, inf = oracle.select(m, 2, tau)
        assert kept.tolist() == [1, 2]
        assert abs(inf[1] / inf[0] - (tau + off)) < 1e-12
        assert oracle.is_boundary(inf, tau) == flagged
