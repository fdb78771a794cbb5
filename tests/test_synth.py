"""The seeded input generator: Philox known answers, determinism, rounding, moments."""
import os

import numpy as np
import pytest

import synth
from synth import configs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _kat():
    rows = []
    with open(os.path.join(GOLDEN, "philox4x32_10_kat.txt")) as fh:
        for line in fh:
            if line.strip() and not line.startswith("#"):
                v = [int(t, 16) for t in line.split()]
                rows.append((v[0:4], v[4:6], v[6:10]))
    return rows


@pytest.mark.parametrize("ctr,key,expected", _kat())
def test_philox_known_answers(ctr, key, expected):
    assert list(synth.philox4x32_10(ctr, key)) == expected


def test_counter_addressing_matches_full_draw():
    full = synth.normal(0, 7, (1001,))
    part = synth.normal(0, 7, (500,), start=333)
    np.testing.assert_array_equal(full[333:833], part)


def test_streams_are_distinct_and_deterministic():
    a = synth.normal(0, 1, (64,))
    assert np.array_equal(a, synth.normal(0, 1, (64,)))
    assert not np.array_equal(a, synth.normal(0, 2, (64,)))
    assert not np.array_equal(a, synth.normal(1, 1, (64,)))


def test_moments():
    z = synth.normal(0, 11, (1 << 20,))
    assert abs(z.mean()) < 5e-3
    assert abs(z.std() - 1.0) < 5e-3
    # fraction beyond 2 sigma of a standard normal is 0.0455
    assert abs(np.mean(np.abs(z) > 2.0) - 0.0455) < 2e-3


def test_storage_rounding_is_round_to_nearest_even():
    z = synth.normal(0, 3, (4096,), std=0.5)
    f32 = synth.normal(0, 3, (4096,), std=0.5, dtype="f32")
    np.testing.assert_array_equal(f32, z.astype(np.float32))
    bits = synth.normal(0, 3, (4096,), std=0.5, dtype="bf16")
    back = (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    # nearest: no other bf16 value is closer
    step = np.abs(back) * 2.0 ** -7
    assert np.all(np.abs(back - z) <= step / 2 * (1 + 1e-12))
    # ties go to even mantissa
    ties = np.array([1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -(1.0 + 2.0 ** -8)])
    tb = synth.round_bf16(ties)
    assert list(tb) == [0x3F80, 0x3F82, 0xBF80]


def test_workload_shapes():
    w = configs.WORKLOADS["tiny_f32"]
    assert configs.make_x(w).shape == (64, 256) and configs.make_x(w).dtype == np.float32
    assert configs.make_w_gate(w).shape == (8, 256, 1024)
    assert configs.make_w_down(w).shape == (8, 1024, 256)
    m = configs.WORKLOADS["mid_bf16"]
    assert configs.make_router(m).dtype == np.uint16
    rows = configs.make_x(m, rows=(10, 20))
    np.testing.assert_array_equal(rows, configs.make_x(m)[10:20])
