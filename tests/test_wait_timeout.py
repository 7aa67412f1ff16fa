"""The kernels' bounded waits on the GPU, without a fault: a probe kernel waits
on an mbarrier that nothing arrives at, gives up after its limit, records
FLARE_ERR_TIMEOUT in the status word and returns.  The host reads the status
(and clears it), and the context then runs the mixer as before.
"""
import time

import numpy as np
import pytest

import oracle
import rank_latent_attention_b200 as flare
from gpu_common import assert_stated, require_cuda, to_dev, to_host
from rank_latent_attention_b200 import inputs

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_context_survives():
    torch = require_cuda()
    L = flare.lib()
    assert flare.flare_check_status() == (0, 0)
    t0 = time.perf_counter()
    assert L.flare_selftest_wait_timeout(50, None) == 0
    assert flare.flare_check_status() == (4, 13)  # FLARE_ERR_TIMEOUT, recorded by the probe
    elapsed = time.perf_counter() - t0
    assert 0.045 <= elapsed < 5.0, elapsed     # it waited its 50 ms, then returned
    assert flare.flare_check_status() == (0, 0)  # reading the status cleared it
    assert L.flare_selftest_wait_timeout(0, None) == 1 and L.flare_selftest_wait_timeout(1001, None) == 1
    # the context still works: a small mixer forward against the oracle
    w = inputs.custom(1, 2, 300, 32, 16, dtype="f32", seed_index=95)
    seeds, K, V = inputs.make_inputs(w)
    Y = flare.flarepp_mix(*(to_dev(x, "f32") for x in (seeds, K, V)))
    assert flare.flare_check_status() == (0, 0)
    _, _, Yo = oracle.flarepp_mix(seeds.astype(np.float64), K.astype(np.float64), V.astype(np.float64))
    assert_stated("after_timeout.Y", to_host(Y), Yo, "f32")
