"""Host test of the parity check that bench.py runs before timing: the
oracle's row-sampled results (O, LSE, dQ) against given outputs, plus the sum
identities of dK and dV.  Outputs computed by the full float64 oracle pass;
outputs with a planted error in any of the five tensors fail."""
import math

import numpy as np
import pytest

import bench
import oracle
from exact_attention_112_b200 import inputs


@pytest.fixture(scope="module")
def case():
    w = inputs.workload("bwd", B=1, H=2, Nq=300, Nk=300, D=64)
    arrs = bench.oracle_sample_setup(w, ["fwd", "bwd"])
    scale = 1.0 / math.sqrt(w["D"])
    o, lse = oracle.fwd(arrs["q"], arrs["k"], arrs["v"], None, True, scale)
    dq, dk, dv = oracle.bwd(arrs["q"], arrs["k"], arrs["v"], arrs["do"], None, True, scale)
    shp = (w["B"], w["H"])
    gpu = {"o": o, "lse": lse, "dq": dq.reshape(*shp, 300, 64), "dk": dk.reshape(*shp, 300, 64),
           "dv": dv.reshape(*shp, 300, 64), "do": arrs["do"]}
    rows = bench.pick_rows(w, 40, boundaries=True)
    ref = {}
    bench.oracle_rows_time(arrs, w, rows, ["fwd", "bwd"], outputs=ref)
    return w, rows, ref, gpu


def test_exact_outputs_pass(case):
    w, rows, ref, gpu = case
    rep = bench.parity_report(w, rows, ref, gpu)
    assert rep["ok"], rep
    assert rep["o_max_abs"] < 1e-12 and rep["dq_rel_to_max"] < 1e-12
    assert rep["sum_dv_rel"] < 1e-12 and rep["sum_dk_rel"] < 1e-12
    assert 0 in rows and 127 in rows and 128 in rows and 299 in rows


@pytest.mark.parametrize("what", ["o", "lse", "dq", "dk", "dv"])
def test_planted_errors_fail(case, what):
    w, rows, ref, gpu = case
    bad = {k: np.array(v) for k, v in gpu.items()}
    t = bad[what]
    if what in ("o", "lse", "dq"):
        t[0, 1, rows[3]] += 0.5                 # one sampled row wrong
    elif what == "dk":
        t[0, 0, 5] += 0.5 * np.abs(t).max()     # a dK row off: its column sum is no longer 0
    else:
        t[0, 1] *= 1.1                          # dV of one head scaled
    rep = bench.parity_report(w, rows, ref, bad)
    assert not rep["ok"], (what, rep)


def test_cpu_baseline_fields():
    """The cpu_baseline leg reports its FLOP rate, the rows per second and the
    whole step's extrapolated time (consistent with each other), and for the
    tiny workload a single-thread figure as well."""
    w = inputs.workload("tiny")
    base, report = bench.cpu_baseline(w, 0.2, ["fwd"])
    assert report is None
    total = sum(bench.flops_of(w, ["fwd"]).values())
    assert base["value"] > 0 and base["rows_per_s"] > 0 and base["cores"] >= 1
    assert math.isclose(base["full_step_s_extrapolated"] * base["value"] * 1e12, total, rel_tol=1e-9)
    assert base["one_thread"]["value"] > 0 and base["one_thread"]["seconds"] > 0
    assert oracle.max_threads() == base["cores"]   # the thread count is restored
