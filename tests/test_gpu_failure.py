"""Failure detection on the GPU without a fault: a bounded wait that nothing
completes gives up, the host reads DSA_ERR_TIMEOUT from the device error
word, and the next calls run normally on the same context."""
import time

import pytest
import torch

import long_context_indexing_lightning_b200 as dsa
import workloads
from long_context_indexing_lightning_b200 import build

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_context_stays_usable():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build.build()
    dsa.lib()
    dsa.get_error(clear=True)
    t0 = time.time()
    dsa.selftest_wait_timeout()
    rc, word = dsa.get_error(clear=True)
    waited = time.time() - t0
    assert rc == 5 and (word & 1), (rc, word)          # DSA_ERR_TIMEOUT
    assert 1.0 < waited < 30.0, waited
    # the context is intact: a normal step runs and reports no error
    wl = workloads.get("decode32k", batch=2, s_max=2048)
    t = workloads.make_inputs(wl, "cuda", seed=1)
    out = dsa.forward(dsa.shape_from_workload(wl), t["q_idx"], t["k_idx"], t["w"], t["q"], t["kv"],
                      t["ctx_len"], t["q_pos0"])
    torch.cuda.synchronize()
    assert torch.isfinite(out.float()).all()
    rc, word = dsa.get_error(clear=True)
    assert rc == 0, word
