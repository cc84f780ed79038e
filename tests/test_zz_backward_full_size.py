"""Backward parity at the sizes the benchmark times (bench.py --workload
bwd_full_s4096 and bwd_sliding_s1024): the same seeded inputs, the library's
forward, then the backward, every gradient compared with the FP64 backward
oracle over all rows at the tolerances derived in tests/test_backward.py."""
import numpy as np
import pytest

import workloads as W
from test_backward import _compare, _dout_bits, _run

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name", ["sliding_s1024", "full_s4096"])
def test_backward_at_bench_size(name):
    w = W.make(name)
    dO = _dout_bits(w.T, 1000 + w.seed)
    got, _ = _run(w, dO)
    _compare(w, dO, got)
