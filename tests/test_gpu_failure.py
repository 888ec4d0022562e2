"""Failure detection on the GPU without a fault: a bounded pipeline wait that
runs out (on a barrier nothing arrives at) reports VDN_INFO_TIMEOUT through
the info word, and the context stays usable for the next pass. Nothing here
traps, asserts or hangs a GPU."""
import time

import pytest
import torch

from frame_wise_delta_b200 import synth, vdn
from test_gpu_parity import TC_SMALL
from vdn_testlib import TOL, device_inputs, oracle_heads, rel, run_forward

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _build():
    from frame_wise_delta_b200 import build
    build.build()
    assert torch.cuda.is_available()


def test_bounded_wait_runs_out_and_the_context_stays_usable():
    info = torch.full((1,), 7, dtype=torch.int32, device="cuda")
    t0 = time.perf_counter()
    vdn.vdn_selftest_wait(info)
    torch.cuda.synchronize()
    dt = time.perf_counter() - t0
    assert int(info.item()) == vdn.VDN_INFO_TIMEOUT
    assert 1.0 < dt < 30.0, dt  # the wait gave up after its 1.5 s limit
    # the next pass runs and matches the oracle
    w = TC_SMALL
    full = synth.generate_all(w)
    fw = run_forward(w, device_inputs(w, full))
    assert int(fw.info.item()) == 0
    ref = oracle_heads(w, full, [(0, 0)])
    assert rel(fw.O[0, 0], ref[(0, 0)]["O"]) <= TOL[w.dtype]


def test_selftest_argument_check():
    with pytest.raises(vdn.VdnError):
        vdn.vdn_selftest_wait(None)
