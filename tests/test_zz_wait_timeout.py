"""The failure path of the kernels' bounded waits, on the GPU.

A diagnostic kernel waits on an mbarrier that nothing arrives at, through the
same wait the prefill kernels use.  The wait must end by its ~2 s limit with
no fault or trap.  The host must read KASCADE_ERR_TIMEOUT from the status word
(once, then clear), and the context must stay usable: a Top-k call afterwards
is bit-exact against the oracle.  The file sorts last, so with -x its few
seconds of waiting come after every other GPU test.
"""
import time

import numpy as np
import pytest
import torch

import oracle as O
from long_context_emitting_b200 import api, binding


@pytest.mark.gpu
@pytest.mark.parametrize("spin", [False, True], ids=["try_wait", "test_wait"])
def test_bounded_wait_gives_up_and_reports(spin):
    api.device_status()  # start from a clear status word
    t0 = time.perf_counter()
    assert api.selftest_wait_timeout(spin) == binding.KASCADE_ERR_TIMEOUT
    elapsed = time.perf_counter() - t0
    assert 1.5 < elapsed < 60.0, elapsed
    assert api.device_status() == binding.KASCADE_OK  # read once, then cleared

    # the context is still usable
    dev = torch.device("cuda")
    g = torch.Generator().manual_seed(17)
    n, k = 1000, 128
    scores = torch.rand(4, n, generator=g)
    lens = torch.full((4,), n, dtype=torch.int32)
    ks = torch.full((4,), k, dtype=torch.int32)
    out = api.topk(scores.to(dev), lens.to(dev), ks.to(dev), k)
    assert api.device_status() == binding.KASCADE_OK
    expect = O.topk_rows(scores.numpy(), lens.tolist(), ks.tolist(), k)
    np.testing.assert_array_equal(out.cpu().numpy(), expect)
