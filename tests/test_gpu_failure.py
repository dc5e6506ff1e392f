"""Failure detection on the GPU without a fault: a bounded device wait that
runs out is reported as FIPA_ERR_DEVICE_TIMEOUT through the handle's status
word, and the context stays usable (the next forward matches the oracle)."""
import time

import numpy as np
import pytest
import torch

import oracle
import workloads
from parity_util import compare, to_device

pytestmark = pytest.mark.gpu


def test_bounded_wait_timeout_is_reported_and_context_survives():
    from protein_structure_models_b200 import Fipa, FipaError, build
    build.build()
    h = Fipa("f32", 0)
    try:
        t0 = time.perf_counter()
        h.selftest_timeout(50)                    # a wait on a barrier nothing completes
        with pytest.raises(FipaError) as ei:
            h.sync_status()
        waited = time.perf_counter() - t0
        assert ei.value.status == 5               # FIPA_ERR_DEVICE_TIMEOUT
        assert "site 63" in str(ei.value)         # the self-test's wait site
        assert 0.04 <= waited < 5.0               # it ended by its own budget
        h.sync_status()                           # the status word was cleared
        # the context and the handle still work: a normal forward, checked
        inp = workloads.make_inputs(workloads.workload(0))
        out = h.forward(to_device(inp, "f32"), eps=inp["eps"], want_attention=False, want_lse=True)
        h.sync_status()
        torch.cuda.synchronize()
        ref = oracle.ipa_forward_dense(inp)
        compare(out, ref, "f32", check_attention=False)
    finally:
        h.close()


def test_selftest_argument_validation():
    from protein_structure_models_b200 import Fipa, FipaError, build
    build.build()
    h = Fipa("f32", 0)
    try:
        for bad in (0, 10001):
            with pytest.raises(FipaError) as ei:
                h.selftest_timeout(bad)
            assert ei.value.status == 1
    finally:
        h.close()
