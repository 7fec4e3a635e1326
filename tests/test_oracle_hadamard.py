"""Pins of the structured (randomized Hadamard) rotation: the oracle's fast transform against the
closed form of the Sylvester-Hadamard matrix, and the rotation input against both."""

from __future__ import annotations

import numpy as np
import pytest

import tq_synth as syn
from oracle import turboquant as otq


def _sylvester_closed_form(d):
    # H_ij = (-1)^popcount(i & j), a textbook identity independent of the recursive construction
    i = np.arange(d)
    pc = np.vectorize(lambda v: bin(int(v)).count("1"))(i[:, None] & i[None, :])
    return np.where(pc % 2 == 0, 1.0, -1.0)


@pytest.mark.parametrize("d", [1, 2, 8, 64, 128])
def test_fast_transform_is_the_sylvester_matrix(d):
    assert np.array_equal(otq.walsh_hadamard(np.eye(d)), _sylvester_closed_form(d))


def test_fast_transform_rejects_other_lengths():
    with pytest.raises(ValueError):
        otq.walsh_hadamard(np.zeros((2, 200)))


@pytest.mark.parametrize("d", [8, 128, 256])
def test_randomized_hadamard_input(d):
    Pi = syn.randomized_hadamard(d).double().numpy()
    # |entries| = 1/sqrt(d); the first row of H is all ones, so it carries the signs
    assert np.allclose(np.abs(Pi), 1 / np.sqrt(d), rtol=1e-7, atol=0)
    s = np.sign(Pi[0])
    want = _sylvester_closed_form(d) * s[None, :] / np.sqrt(d)
    assert np.allclose(Pi, want, rtol=0, atol=1e-7)
    assert np.allclose(Pi @ Pi.T, np.eye(d), rtol=0, atol=1e-6)
    # the fast form and the dense product agree on random rows
    u = np.random.default_rng(1).standard_normal((5, d))
    assert np.allclose(otq.structured_rotate(u, s), u @ want.T, rtol=0, atol=1e-12)
    assert np.mean(s > 0) not in (0.0, 1.0)


def test_encoding_with_structured_rotation_matches_dense():
    # the oracle's encoder with the Hadamard input: y = Pi u equals the fast transform of s * u
    d = 128
    Pi = syn.randomized_hadamard(d).double().numpy()
    s = np.sign(Pi[0])
    x = np.random.default_rng(2).standard_normal((64, d))
    e = otq.quantize(x, Pi, np.array([-0.07, -0.02, 0.02, 0.07]))
    u = x / np.linalg.norm(x, axis=1, keepdims=True)
    assert np.allclose(e["y"], otq.structured_rotate(u, s), rtol=0, atol=1e-6)
