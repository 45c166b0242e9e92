"""Failure path of the bounded device waits, exercised without a GPU fault.

A diagnostic kernel waits on an mbarrier that nothing arrives on; its bounded
wait gives up after 2 ms and records the timeout.  The host must read
QS_ERR_TIMEOUT through qs_device_error, the word must be cleared by that read,
and the context must stay usable (a real layer runs correctly afterwards).
"""

import time

import numpy as np
import pytest
import torch

import bit_quantized_linear_hadamard_b200 as qs
from bit_quantized_linear_hadamard_b200 import build as qs_build
from bit_quantized_linear_hadamard_b200 import inputs as I
from oracle import qs_oracle as O

pytestmark = pytest.mark.gpu

QS_ERR_TIMEOUT = 7


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    qs_build.build()
    qs.load()


def test_bounded_wait_reports_timeout_and_context_survives():
    assert qs.qs_device_error() == 0
    t0 = time.perf_counter()
    qs.qs_selftest_timeout(2000)
    assert qs.qs_device_error() == QS_ERR_TIMEOUT
    assert time.perf_counter() - t0 < 5.0, "the wait must give up after its bound"
    assert qs.qs_device_error() == 0, "reading the error word clears it"
    d = I.make_layer(I.TINY)
    wp, ws = qs.pack_weights(d["w"].cuda(), 4)
    out = qs.linear(d["x"].cuda(), wp, ws, d["bias"].cuda(), 4, 1.0)
    torch.cuda.synchronize()
    r = O.qlinear(I.bf16_bits(d["x"]), I.bf16_bits(d["w"]), I.bf16_bits(d["bias"]), 4, 1.0)
    assert np.array_equal(out.view(torch.int16).cpu().numpy().view(np.uint16), r["out"])
    assert qs.qs_device_error() == 0
