"""Pins of the oracle's packed codes and lookup-table product (CPU only).

The consumer of (C, Q): "GuidedQuant" blog post, LNQ section (LNQ runs on SqueezeLLM's CUDA
kernel), and the aitopics "squeezellm" tag page (SqueezeLLM and GANQ abstracts: single-batch
inference is memory-bound, weights as low-bit indices into a lookup table). The packing format is
reading R6 of oracle/lnq_oracle.c.
"""
import json
import os

import numpy as np
import pytest

from oracle import oracle as orc

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "lut_pack.json")


def test_pack_matches_hand_derived_words():
    cases = json.load(open(GOLDEN))["cases"]
    for c in cases:
        Q = np.array([c["codes"]], dtype=np.uint8)
        P = orc.pack_codes(Q, c["bits"])
        assert P.shape == (1, len(c["words"]))
        np.testing.assert_array_equal(P[0], np.array(c["words"], dtype=np.uint32))


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
@pytest.mark.parametrize("d_in", [1, 7, 10, 31, 32, 33, 100, 257])
def test_pack_unpack_roundtrip_and_zero_padding(bits, d_in):
    rng = np.random.default_rng(bits * 1000 + d_in)
    Q = rng.integers(0, 1 << bits, size=(5, d_in), dtype=np.uint8)
    P = orc.pack_codes(Q, bits)
    per = 32 // bits
    assert P.shape == (5, (d_in + per - 1) // per)
    np.testing.assert_array_equal(orc.unpack_codes(P, d_in, bits), Q)
    # bits above per * bits and past the row's last code are zero
    used = np.zeros(P.shape[1], dtype=np.uint64)
    for w in range(P.shape[1]):
        n = min(per, d_in - w * per)
        used[w] = (1 << (n * bits)) - 1
    assert np.all((P.astype(np.uint64) & ~used) == 0)


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_lut_product_equals_dense_product(bits):
    """y = x W^T with W^ = C[Q] formed densely and multiplied by numpy."""
    rng = np.random.default_rng(bits)
    d_out, d_in, nb, m = 9, 77, 3, 1 << bits
    C = rng.standard_normal((d_out, m))
    Q = rng.integers(0, m, size=(d_out, d_in), dtype=np.uint8)
    x = rng.standard_normal((nb, d_in))
    W_hat = np.take_along_axis(C, Q.astype(np.int64), axis=1)
    np.testing.assert_allclose(orc.lut_gemv(x, C, Q), x @ W_hat.T, rtol=1e-12, atol=1e-12)


def test_lut_product_integer_codebook_is_exact():
    """With c_k = k and integer activations every sum is an exact integer: y = x Q^T."""
    rng = np.random.default_rng(7)
    Q = rng.integers(0, 16, size=(6, 50), dtype=np.uint8)
    x = rng.integers(-5, 6, size=(2, 50)).astype(np.float64)
    C = np.tile(np.arange(16.0), (6, 1))
    np.testing.assert_array_equal(orc.lut_gemv(x, C, Q), x @ Q.astype(np.float64).T)
