"""The synthetic input recipes match their stated laws (these are the inputs both the CUDA path and
the oracle receive): seeded and reproducible, shapes and dtypes, and the distributional properties
each workload's description names."""

from __future__ import annotations

import numpy as np
import torch

import tq_synth as syn


def test_rotation_and_sketch():
    Pi, S = syn.rotation(64), syn.sketch(64)
    assert Pi.dtype == torch.float32 and S.dtype == torch.float32
    P = Pi.double().numpy()
    assert np.allclose(P @ P.T, np.eye(64), atol=1e-6)
    assert torch.equal(Pi, syn.rotation(64)) and not torch.equal(Pi, syn.rotation(64, seed=9))
    s = S.double().numpy().ravel()
    assert abs(s.mean()) < 0.05 and abs(s.std() - 1.0) < 0.05


def test_nn_inputs_law():
    db, qs = syn.nn_inputs(20000, 300, 200)
    assert db.shape == (20000, 200) and qs.shape == (300, 200) and db.dtype == torch.float32
    assert torch.allclose(db.norm(dim=1), torch.ones(20000), atol=1e-5)
    assert torch.allclose(qs.norm(dim=1), torch.ones(300), atol=1e-5)
    # one anisotropic law for both: per-dimension spread tracks the seeded std ~ U[0.2, 2]
    sig = 0.2 + 1.8 * torch.rand(200, generator=torch.Generator().manual_seed(10), dtype=torch.float32)
    spread = db.std(dim=0)
    corr = np.corrcoef(spread.numpy(), sig.numpy())[0, 1]
    assert corr > 0.99
    ratio = spread / sig
    assert float(ratio.std() / ratio.mean()) < 0.05
    # the database and the queries are different draws of that law
    assert not torch.allclose(db[:300], qs)
    db2, _ = syn.nn_inputs(20000, 300, 200)
    assert torch.equal(db, db2)

