"""The row-block process pool that the full-size GPU tests use for the
oracle's per-row work gives exactly the serial oracle's results (row order,
every array), on small inputs.  No GPU is involved."""

import numpy as np
import torch

import oracle_pool as P
from bit_quantized_linear_hadamard_b200 import inputs as I
from oracle import bgr_oracle as B
from oracle import sd4_oracle as S


def _bits(rows, cols, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    return I.bf16_bits((torch.randn(rows, cols, generator=g) * scale).to(torch.bfloat16))


def test_bgr_pack_matches_serial():
    wb = _bits(37, 384, 1, 0.02)
    got = P.bgr_pack_weights(wb, 4, 16, 3)
    want = B.pack_weights_bgr(wb, 4, 16, 3)
    assert len(got) == 3
    for g, w in zip(got, want):
        assert g.dtype == w.dtype and np.array_equal(g, w)


def test_sd4_quantize_and_decompose_match_serial():
    xb = _bits(29, 256, 2)
    got = P.sd4_quantize_rows(xb)
    want = S.quantize_rows(xb)
    for g, w in zip(got, want):
        assert np.array_equal(g, w)
    rows = [0, 3, 11, 28]
    gd = P.sd4_decompose_rows(xb[rows])
    wd = S.decompose_rows(xb, rows)
    assert gd.keys() == wd.keys()
    for k in wd:
        assert np.array_equal(gd[k], wd[k]), k
