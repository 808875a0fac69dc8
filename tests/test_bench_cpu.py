"""The CPU baseline of bench.py (the oracle timed on the host): its sampling and the throughput it reports,
without a GPU."""
import math

import bench
import workloads


def _gems(make):
    return [(g, 0) for g in make()]


def test_per_tensor_quantisation_is_made_once_and_counted_in_every_run():
    s = bench.OracleSample(_gems(workloads.tiny))  # tiny quantises per tensor
    t1, ops1, fixed1 = s.run(0.5)
    t2, ops2, fixed2 = s.run(0.25)
    assert fixed1 > 0 and fixed2 == fixed1  # measured once, the same time counted again
    assert t1 >= fixed1 and t2 >= fixed2
    assert ops1 > ops2 > 0
    assert len(s.qcache) == 2  # A and B


def test_rate_scales_the_sample_to_the_whole_products():
    s = bench.OracleSample(_gems(workloads.tiny))
    frac = 0.25
    t, ops, fixed = s.run(frac)
    full = sum(2.0 * g.M * g.N * g.K for g in workloads.tiny())
    assert s.full_ops() == full
    want = full / (fixed + (t - fixed) / frac ** 2)
    assert math.isclose(s.rate(t, ops, fixed, frac), want, rel_tol=1e-12)
    # without per-tensor work the rate is the sample's own
    assert s.rate(2.0, 10.0, 0.0, frac) == 5.0


def test_per_row_workloads_have_no_fixed_part():
    g = workloads.q_proj()[0]
    s = bench.OracleSample([(g, 0)])
    _, ops, fixed = s.run(1.0 / 256)
    assert fixed == 0.0 and ops > 0
