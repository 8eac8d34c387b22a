"""Failure detection on the GPU without a fault: every kernel's mbarrier
waits are bounded.  A wait that nothing completes gives up after about a
second, sets the device error word and returns; the host reads it as
ABATTN_ERR_TIMEOUT and the CUDA context stays usable."""
import ctypes
import math
import time

import numpy as np
import pytest
import torch

import oracle
from block_sparse_attention_12_b200 import abi, build

pytestmark = pytest.mark.gpu


def test_bounded_wait_gives_up_and_the_context_survives():
    S = ctypes.CDLL(build.build_selftest())
    f = S.abattn_selftest_stalled_wait
    f.restype, f.argtypes = ctypes.c_int, [ctypes.POINTER(ctypes.c_int), ctypes.c_void_p]
    waited = ctypes.c_int(-2)
    t0 = time.monotonic()
    rc = f(ctypes.byref(waited), None)
    dt = time.monotonic() - t0
    assert rc == abi.ERR_TIMEOUT, abi.strerror(rc)
    assert waited.value == 0  # the kernel ran and its wait gave up
    assert 0.2 < dt < 30.0, dt  # the limit is about 2e9 SM cycles
    # the same process and context still run the library's kernels
    g = torch.Generator().manual_seed(7)
    Qc, Kc, Vc = (torch.randn(1, 1, 300, 64, generator=g).to(torch.bfloat16) for _ in range(3))
    O, lse = abi.dense_forward(Qc.cuda(), Kc.cuda(), Vc.cuda())
    assert abi.check() is None
    Oo, lo = oracle.dense(Qc[0, 0], Kc[0, 0], Vc[0, 0], 1 / math.sqrt(64))
    np.testing.assert_allclose(O[0, 0].float().cpu().numpy(), Oo, atol=2e-2)
    np.testing.assert_allclose(lse[0, 0].cpu().numpy(), lo, atol=2e-3, rtol=1e-4)
