"""qs_linear_noalloc: the layer on the library's own fixed scratch buffer.

For callers that cannot allocate device memory when they run the layer (a
runtime that owns the whole memory pool, a plugin interface without a
workspace, a loop that cannot afford an allocation per call), the library
offers qs_linear_noalloc, which takes only inputs and outputs and uses a
buffer kept in the library's device memory.  Here it is called through the C
ABI, twice in a row with different inputs, and compared with qs_linear on a
caller-provided workspace (the tests' tolerance: 1 bf16 ulp; expected
bit-identical).  Sizes beyond the buffer are rejected.

The file name sorts last so that a run stopping at the first failure has run
every other test before this one.
"""

import numpy as np
import pytest
import torch

import bit_quantized_linear_hadamard_b200 as qs
from bit_quantized_linear_hadamard_b200 import binding
from bit_quantized_linear_hadamard_b200 import build as qs_build
from bit_quantized_linear_hadamard_b200 import inputs as I

pytestmark = pytest.mark.gpu

QS_ERR_RANGE = 5


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    qs_build.build()
    qs.load()


def _ordered(b):
    b = b.astype(np.int32)
    mag = b & 0x7FFF
    return np.where(b & 0x8000, -mag, mag)


def _bits(t):
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


@pytest.mark.parametrize("bits,alpha", [(4, 0.9), (8, 1.0)])
def test_noalloc_matches_qs_linear_on_two_calls(bits, alpha):
    K, N = 640, 528
    d0 = I.make_shape(seed=31, M=300, K=K, N=N, bits=bits, alpha=alpha, outlier_factor=50.0)
    d1 = I.make_shape(seed=32, M=129, K=K, N=N, bits=bits, alpha=alpha, outlier_factor=50.0)
    w, b = d0["w"].cuda(), d0["bias"].cuda()
    wp, ws = qs.pack_weights(w, bits)
    for d in (d0, d1):
        x = d["x"].cuda()
        M = x.shape[0]
        want = qs.linear(x, wp, ws, b, bits, alpha)
        got = torch.full((M, N), -1.0, dtype=torch.bfloat16, device="cuda")
        binding.qs_linear_noalloc(x, M, K, alpha, wp, ws, b, N, bits, got)
        torch.cuda.synchronize()
        diff = np.abs(_ordered(_bits(got)) - _ordered(_bits(want)))
        assert diff.max() <= 1, "within 1 bf16 ulp of qs_linear"
        assert (diff == 0).all(), "same kernels, same arithmetic: bit-identical"
    assert qs.qs_device_error() == 0


def test_noalloc_rejects_sizes_beyond_its_buffer():
    K, bits = 5120, 4
    m_max = 0
    while qs.qs_linear_workspace_bytes(m_max + 1, K, bits) <= binding.QS_NOALLOC_SCRATCH_BYTES:
        m_max += 1
    assert m_max == 3271
    L = binding.load()
    x = torch.zeros((m_max + 1, K), dtype=torch.bfloat16, device="cuda")
    wp = torch.zeros((16, K // 2), dtype=torch.uint8, device="cuda")
    ws = torch.ones((16,), dtype=torch.float32, device="cuda")
    out = torch.empty((m_max + 1, 16), dtype=torch.bfloat16, device="cuda")
    st = L.qs_linear_noalloc(binding._p(x), m_max + 1, K, 1.0, binding._p(wp), binding._p(ws), None,
                             16, bits, binding._p(out), binding._s(None))
    assert st == QS_ERR_RANGE
