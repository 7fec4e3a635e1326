"""Failure detection on the GPU without a GPU fault: a bounded wait that runs out.

Every mbarrier wait in the library's kernels gives up after a bounded number of tries and records a
timeout in the call's status word, which tq_workspace_status reports as TQ_ERR_DEVICE. The test hook
tq_debug_stall_consumers makes the softmax.V kernel's consumer warps wait on a barrier that nothing
completes, for a few tries: the wait must run out, the call's status must say so, the copies in flight
must still land (the copy thread drains them at the full limit), and the context must stay usable, so
that the same call right after gives a clean status and the oracle's result.
"""

from __future__ import annotations

import math

import numpy as np
import pytest
import torch

import tq_synth as syn
from oracle import codebook as ocb
from tests import _parity as par

pytestmark = pytest.mark.gpu

cuda_ok = torch.cuda.is_available()
if cuda_ok:
    import kv_cache_vector_quantize_b200 as tqb


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not cuda_ok:
        pytest.skip("needs a CUDA device")


def test_consumer_wait_runs_out_and_is_reported():
    d, bits, H, T = 128, 3, 2, 3000
    dev = torch.device("cuda")
    Pi = syn.rotation(d)
    cv = ocb.fit_codebook(d, bits)[0]
    Pig, cvg = Pi.to(dev), torch.from_numpy(cv).to(dev)
    v = syn.lognormal_sphere((1, H, T, d), 95, dtype=torch.bfloat16, device=dev)
    vc = tqb.PackedCache.empty(d, bits, False, 1, H, T)
    tqb.tq_quantize_append(vc, v, 0, Pig, None, cvg)
    lg = 3.0 * syn.gaussian((1, H, T), 96, device=dev)
    sc = 1.0 / math.sqrt(d)
    ws = torch.zeros(max(256, tqb.tq_attend_workspace_size(vc, H, T)), dtype=torch.uint8, device=dev)
    tqb.tq_attend_v(vc, lg, sc, T, Pig, cvg, workspace=ws)
    tqb.tq_workspace_status(ws)                       # a normal call: clean
    tqb.tq_debug_stall_consumers(64)
    try:
        tqb.tq_attend_v(vc, lg, sc, T, Pig, cvg, workspace=ws)
        with pytest.raises(tqb.TQError) as e:
            tqb.tq_workspace_status(ws)
        assert e.value.status == tqb.TQ_ERR_DEVICE
        assert "0x00000002" in tqb.tq_last_error()    # the timeout bit, no other
    finally:
        tqb.tq_debug_stall_consumers(0)
    tqb.tq_workspace_status(ws)                       # read and cleared: clean again
    # the context is intact: the same call gives a clean status and the oracle's softmax.V
    out = tqb.tq_attend_v(vc, lg, sc, T, Pig, cvg, workspace=ws)
    tqb.tq_workspace_status(ws)
    rec = par.as_u32(vc.records.cpu().numpy())
    for h in range(H):
        par.check_attend(out[0, h:h + 1].cpu().numpy(), lg[0, h:h + 1].cpu().numpy().astype(np.float64), sc,
                         Pi.numpy(), cv, rec[0, h], vc.norm[0, h].cpu().numpy(), d, bits)
