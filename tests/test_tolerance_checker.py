"""Pins of the parity checker itself (no GPU).

Every GPU parity test and the smoke check decide pass/fail through
oracle.check_tolerance, the element-wise rule |c - ref| <= 1e-2 |ref| + 1e-3 rms(ref)
(the "<1% relative error against a higher-precision reference" of the DeepGEMM
library page, 2kiu.com/news/5461879 §6, with an absolute floor scaled by the
output's RMS).  These tests feed it constructed pairs whose outcome is fixed by
hand arithmetic, so that a slip in the checker -- the RMS taken over the wrong
values, the absolute term scaled by |ref|, the comparison inverted, NaN let through,
the bad elements miscounted -- fails here instead of turning every parity test green.
"""
import numpy as np
import pytest

import oracle
import parity

# ref chosen so that every figure below is exact in binary and by hand:
# mean of squares = (300^2 + 400^2 + 0 + 0) / 4 = 62500, so rms = 250;
# bounds: 3 + 0.25, 4 + 0.25, 0.25, 0.25 (mean |ref| would be 175, not 250).
REF = np.array([300.0, -400.0, 0.0, 0.0])
BOUND = np.array([3.25, 4.25, 0.25, 0.25])


def _with(i, delta):
    c = REF.copy()
    c[i] += delta
    return c


@pytest.mark.parametrize("i", range(4))
@pytest.mark.parametrize("sign", [1.0, -1.0])
def test_just_inside_passes_just_outside_fails(i, sign):
    ok, nbad, _ = oracle.check_tolerance(_with(i, sign * 0.9999 * BOUND[i]), REF)
    assert ok and nbad == 0
    ok, nbad, ratio = oracle.check_tolerance(_with(i, sign * 1.0001 * BOUND[i]), REF)
    assert not ok and nbad == 1
    assert ratio == pytest.approx(1.0001, rel=1e-9)


def test_exact_match_passes_with_ratio_zero():
    ok, nbad, ratio = oracle.check_tolerance(REF.copy(), REF)
    assert ok and nbad == 0 and ratio == 0.0


def test_rms_is_root_mean_square_of_ref():
    # 0.24 is inside 1e-3 * 250 but outside 1e-3 * 175 (mean |ref|) and outside 0
    # (an absolute term scaled by |ref| instead of the RMS)
    ok, _, _ = oracle.check_tolerance(_with(2, 0.24), REF)
    assert ok
    # the RMS is that of ref, not of c: a large error in c must not widen the bound
    ok, nbad, _ = oracle.check_tolerance(_with(0, 1000.0), REF)
    assert not ok and nbad == 1


def test_explicit_rms_overrides_default():
    # rms = 1000 -> the floor is 1.0 on every element
    ok, _, _ = oracle.check_tolerance(_with(3, 0.99), REF, rms=1000.0)
    assert ok
    ok, nbad, _ = oracle.check_tolerance(_with(3, 1.01), REF, rms=1000.0)
    assert not ok and nbad == 1
    # and a smaller explicit rms tightens it: 0.2 > 1e-3 * 100
    ok, _, _ = oracle.check_tolerance(_with(3, 0.2), REF, rms=100.0)
    assert not ok


@pytest.mark.parametrize("bad", [np.nan, np.inf, -np.inf])
def test_non_finite_output_fails(bad):
    c = REF.copy()
    c[1] = bad
    ok, nbad, _ = oracle.check_tolerance(c, REF)
    assert not ok and nbad == 1


def test_counts_bad_elements_exactly():
    c = REF + np.array([3.3, -4.3, 0.0, 0.3])  # elements 0, 1, 3 outside
    ok, nbad, _ = oracle.check_tolerance(c, REF)
    assert not ok and nbad == 3
    # the same errors on a larger array: only those three are counted
    big_ref = np.concatenate([REF, np.zeros(996)])
    big_c = np.concatenate([c, np.zeros(996)])
    rms = 250.0 * np.sqrt(4 / 1000)  # = 15.811...; floor 0.0158
    ok, nbad, _ = oracle.check_tolerance(big_c, big_ref)
    assert not ok and nbad == 3
    assert np.sqrt(np.mean(big_ref ** 2)) == pytest.approx(rms)


def test_shapes_are_element_by_element():
    ref2 = REF.reshape(2, 2)
    c2 = ref2.copy()
    c2[1, 1] = 0.3  # the fourth element, bound 0.25
    ok, nbad, _ = oracle.check_tolerance(c2, ref2)
    assert not ok and nbad == 1


def test_parity_check_rejects_a_two_percent_error_in_one_element():
    """A correct oracle output perturbed by 2% in one element must fail the helper
    the GPU parity tests call."""
    rng = np.random.default_rng(7)
    qa = rng.integers(0, 0x7F, size=(128, 256), dtype=np.uint8)
    qb = rng.integers(0, 0x7F, size=(128, 256), dtype=np.uint8)
    qa[qa == 0x7F] = 0
    qb[qb == 0x7F] = 0
    sa = np.full((1, 2), 0.5, np.float32)
    sb = np.full((1, 2), 0.25, np.float32)
    ref = oracle.gemm_ref(qa, sa, qb, sb)
    rms = float(np.sqrt(np.mean(ref * ref)))
    c = oracle.bf16_bits_to_double(oracle.bf16_from_double(ref))
    parity.check(c, ref, rms, "unperturbed")  # the correct output passes
    i, j = np.unravel_index(np.argmax(np.abs(ref)), ref.shape)
    c[i, j] = ref[i, j] * 1.02
    with pytest.raises(AssertionError):
        parity.check(c, ref, rms, "perturbed")
