"""Pins for the oracle's scalar building blocks: exp_spec and the canonical
fp32 reductions.  Each check compares against something other than the
oracle itself: libm in fp64, exact fp64 sums with their forward error
bound, and hand-derived fp32 cases whose result depends on the exact
evaluation order the oracle header states."""
import math

import numpy as np
import pytest

U32 = 2.0 ** -24  # unit roundoff of fp32


def _ulp_dist(a: np.ndarray, b: np.ndarray) -> np.ndarray:
    ia = a.view(np.int32).astype(np.int64)
    ib = b.view(np.int32).astype(np.int64)
    return np.abs(ia - ib)


def test_exp_spec_within_2ulp_of_libm(oracle_lib):
    # dense grid over the softmax domain plus random points
    rng = np.random.default_rng(123)
    xs = np.concatenate([
        np.linspace(-87.0, 0.0, 1_000_001, dtype=np.float32),
        (-87.0 * rng.random(200_000)).astype(np.float32),
        -np.float32(2.0) ** -np.arange(1, 40, dtype=np.float32),
    ])
    ys = oracle_lib.exp_spec(xs)
    ref = np.exp(xs.astype(np.float64)).astype(np.float32)  # correctly rounded to fp32
    assert _ulp_dist(ys, ref).max() <= 2


def test_exp_spec_special_values(oracle_lib):
    e = oracle_lib.exp_spec(np.array([0.0, -0.0, -87.0, -87.0001, -88.0, -1e30], np.float32))
    assert e[0] == 1.0 and e[1] == 1.0
    assert e[2] > 0 and np.isfinite(e[2]) and e[2] >= np.finfo(np.float32).tiny
    assert e[3] == 0.0 and e[4] == 0.0 and e[5] == 0.0
    # exp(-ln2 * j) is 2^-j up to rounding of the argument
    xs = np.array([-math.log(2.0) * j for j in range(1, 30)], np.float32)
    ref = np.exp(xs.astype(np.float64)).astype(np.float32)
    assert _ulp_dist(oracle_lib.exp_spec(xs), ref).max() <= 2


def test_exp_spec_monotone(oracle_lib):
    xs = np.sort(np.linspace(-87.0, 0.0, 300_001, dtype=np.float32))
    ys = oracle_lib.exp_spec(xs)
    assert np.all(np.diff(ys) >= 0)


@pytest.mark.parametrize("d", [8, 256, 264, 2048, 4096])
def test_canon_dot_forward_error_bound(oracle_lib, d):
    rng = np.random.default_rng(d)
    for _ in range(20):
        a = rng.standard_normal(d).astype(np.float32)
        b = (rng.standard_normal(d) * 0.02).astype(np.float32)
        got = float(oracle_lib.canon_dot(a, b))
        exact = float(np.dot(a.astype(np.float64), b.astype(np.float64)))
        n = -(-d // 256) * 8 + 5          # longest chain of roundings
        gamma = n * U32 / (1 - n * U32)
        bound = gamma * float(np.abs(a.astype(np.float64) * b).sum())
        assert abs(got - exact) <= bound


def test_canon_dot_lane_accumulates_before_butterfly(oracle_lib):
    # lane 0 holds 2^24 (j=0); lane 1 holds 1 + 1 (j=8, j=9).  The lane sums
    # first (1 + 1 = 2), then the butterfly adds 2^24 + 2 exactly.  A plain
    # left-to-right sum would give 2^24 (each +1 is lost to rounding).
    a = np.zeros(256, np.float32)
    b = np.ones(256, np.float32)
    a[0] = 2.0 ** 24
    a[8] = 1.0
    a[9] = 1.0
    assert float(oracle_lib.canon_dot(a, b)) == 2.0 ** 24 + 2.0


def test_canon_dot_butterfly_pairs_lane_l_with_l_xor_16_first(oracle_lib):
    # lane 0 = 2^24, lane 16 = 1, lane 1 = 1.  Step o=16 forms 2^24 + 1 -> 2^24
    # (tie to even) before lane 1 is reached, so the result is 2^24.  Pairing
    # lanes 16 and 1 first would give 2^24 + 2.
    a = np.zeros(256, np.float32)
    b = np.ones(256, np.float32)
    a[0] = 2.0 ** 24
    a[8 * 16] = 1.0
    a[8 * 1] = 1.0
    assert float(oracle_lib.canon_dot(a, b)) == 2.0 ** 24


def test_canon_dot_uses_fused_multiply_add(oracle_lib):
    # acc = -(1 + 2^-11); then fma((1 + 2^-12), (1 + 2^-12), acc) = 2^-24
    # exactly, while a rounded product followed by an add gives 0.
    a = np.zeros(256, np.float32)
    b = np.zeros(256, np.float32)
    a[0], b[0] = -(1.0 + 2.0 ** -11), 1.0
    a[1] = b[1] = 1.0 + 2.0 ** -12
    assert float(oracle_lib.canon_dot(a, b)) == 2.0 ** -24


def test_canon_dot_chunk_order(oracle_lib):
    # lane 0 owns j = 0..7 and j = 256..263, chunk c=0 before c=1:
    # a[0] = 2^24, a[256] = 1, a[257] = 1 -> (2^24 + 1) + 1 = 2^24 in order.
    a = np.zeros(512, np.float32)
    b = np.ones(512, np.float32)
    a[0] = 2.0 ** 24
    a[256] = 1.0
    a[257] = 1.0
    assert float(oracle_lib.canon_dot(a, b)) == 2.0 ** 24
    # and the reverse placement keeps the two ones together first
    a2 = np.zeros(512, np.float32)
    a2[0] = 1.0
    a2[1] = 1.0
    a2[256] = 2.0 ** 24
    assert float(oracle_lib.canon_dot(a2, b)) == 2.0 ** 24 + 2.0


def test_canon_sum_bound_and_layout(oracle_lib):
    rng = np.random.default_rng(5)
    for n in (1, 16, 31, 32, 33, 128, 256):
        q = rng.random(n).astype(np.float32)
        got = float(oracle_lib.canon_sum(q))
        exact = float(q.astype(np.float64).sum())
        m = -(-n // 32) + 5
        assert abs(got - exact) <= m * U32 / (1 - m * U32) * exact
    # lane l holds q[l], q[l+32], ...: q[0] = 2^24, q[32] = 1, q[64] = 1 are
    # all lane 0 and summed in index order -> 2^24 before the butterfly
    q = np.zeros(96, np.float32)
    q[0], q[32], q[64] = 2.0 ** 24, 1.0, 1.0
    assert float(oracle_lib.canon_sum(q)) == 2.0 ** 24
    q = np.zeros(96, np.float32)
    q[0], q[32], q[64] = 1.0, 1.0, 2.0 ** 24
    assert float(oracle_lib.canon_sum(q)) == 2.0 ** 24 + 2.0
