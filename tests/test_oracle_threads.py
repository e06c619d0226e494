"""The OpenMP build of the oracle (timed as the CPU baseline on all host cores) computes
exactly what the one-thread checker computes: same per-atom arithmetic, per-thread
scratch, pooled sums still accumulated in ascending atom order."""
import numpy as np
import pytest

import oracle
from sparse_windowed_atom_b200 import workloads
from tests.oracle_cases import from_workload


@pytest.mark.parametrize("style,stage", [("af3", "encoder"), ("esmfold2", "decoder"),
                                         ("esmfold2", "encoder"), ("af3", "decoder")])
def test_openmp_build_is_bit_identical(style, stage):
    w = workloads.make_inputs(workloads.tiny_spec(style, stage, A=200, T=30), seed=31)
    case = from_workload(w)
    args = dict(eps=case["eps"], style=style, stage=stage, radius=case["radius"])
    sel = np.zeros((2, 200), bool)
    sel[:, ::3] = True
    for qs in (None, sel):
        one = oracle.windowed_atom_attention(case["activations"], case["parameters"],
                                             case["masks"], case["structure"], query_select=qs,
                                             threads="one", **args)
        many = oracle.windowed_atom_attention(case["activations"], case["parameters"],
                                              case["masks"], case["structure"], query_select=qs,
                                              threads="all", **args)
        for k in one:
            np.testing.assert_array_equal(one[k], many[k], err_msg=k)


def test_thread_counts():
    assert oracle.threads_used("one") == 1
    assert oracle.threads_used("all") >= 1
