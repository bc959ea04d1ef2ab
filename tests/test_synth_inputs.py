"""The seeded generator: reproducible, counter-based (any slice can be regenerated alone) and
standard normal in distribution."""
import numpy as np

import synth_inputs as si


def test_splitmix64_reference_values():
    # splitmix64 from state 0: the published first outputs of the sequence
    out = si.splitmix64(0, 0, 3)
    assert [hex(int(v)) for v in out] == ["0xe220a8397b1dcdaf", "0x6e789e6aa1b965f4", "0x6c45d188009454f"]


def test_counter_based_slices():
    full = si.splitmix64(1234, 0, 100)
    np.testing.assert_array_equal(full[37:61], si.splitmix64(1234, 37, 24))


def test_normal_moments_and_determinism():
    a = si.normal((1 << 18,), 2001, np.float64)
    assert abs(a.mean()) < 0.01 and abs(a.std() - 1) < 0.01
    np.testing.assert_array_equal(a, si.normal((1 << 18,), 2001, np.float64))
    assert not np.array_equal(a[:100], si.normal((100,), 2002, np.float64))


def test_workloads_are_consistent():
    for w in si.WORKLOADS.values():
        for _, s in w.attention:
            assert s.dh in (40, 64, 80, 160)
        for _, g in w.group_norm:
            assert g.C % g.groups == 0
    assert si.WORKLOADS[2].attention[0][1].flops == 42949672960
