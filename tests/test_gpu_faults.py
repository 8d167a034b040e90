"""Failure handling on the GPU without a GPU fault.

A wait that runs out records DPO_ERR_TIMEOUT and returns instead of hanging;
bad target tokens are reported and scored zero; the context stays usable."""
import time

import numpy as np
import pytest

from preference_alignment_b200 import libdpo
from preference_alignment_b200 import workloads as WL

from dpo_harness import DeviceWorkload, np64

pytestmark = pytest.mark.gpu


def test_bounded_wait_runs_out_and_reports_timeout():
    assert libdpo.check() == libdpo.OK
    t0 = time.time()
    libdpo.selftest_wait_timeout(200)
    st = libdpo.check()
    dt = time.time() - t0
    assert st == libdpo.ERR_TIMEOUT
    assert 0.15 < dt < 10.0
    assert libdpo.check() == libdpo.OK          # the read cleared it
    # the context is still usable: a forward runs and is correct enough to compare
    w = WL.make_custom(R=2, L=64, d=64, V=300, dtype="bf16", seed=51, prompt_range=(1, 20))
    dw = DeviceWorkload(w)
    a = dw.forward(dw.W, want_grad=False)[0]
    b = dw.forward(dw.W, want_grad=False)[0]
    assert libdpo.check() == libdpo.OK
    assert np.array_equal(np64(a), np64(b))
