"""Failure detection without a GPU fault: a wait that nothing satisfies runs out, the
kernel records a timeout and returns, the host reads HEAL_ERR_TIMEOUT, and the context
keeps working (a GEMM right after is still exact)."""
import time

import numpy as np
import pytest
import torch

import error_compensated_gemm_b200 as heal
import synthetic
from oracle import gemm as G
from tests.gpu_helpers import dev, gemm

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_context_survives():
    dev()
    torch.cuda.synchronize()
    assert heal.heal_get_device_status() == heal.HEAL_OK
    t0 = time.time()
    heal.heal_probe_wait_timeout(200)
    st = heal.heal_get_device_status()
    elapsed = time.time() - t0
    assert st == heal.HEAL_ERR_TIMEOUT
    assert 0.15 < elapsed < 5.0
    assert heal.heal_get_device_status() == heal.HEAL_OK          # cleared by the read
    A, B = synthetic.gemm_square(256, seed=0)
    C = gemm(A.numpy(), B.numpy())
    assert G.normwise_rel_err(C, G.gemm_ref(A.numpy(), B.numpy())) <= 1e-6
