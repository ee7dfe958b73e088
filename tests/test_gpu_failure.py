"""Failure detection on the GPU without a fault: a bounded wait that runs out.

Every pipeline wait of the library's kernels gives up after a time limit, sets the context's
device error word and returns; colibri_sync_status reports COLIBRI_ERR_TIMEOUT.  The self-test
entry point waits on a device barrier that nothing ever completes, with a 20 ms limit, so the
whole path runs: the wait gives up, the status is reported once and cleared, and the context
keeps working.
"""
import pytest
import torch

import inputgen
import sparse_expert_ffn_router_b200 as colibri
from tests import gpu_harness as H

pytestmark = pytest.mark.gpu

TIMEOUT = -6


@pytest.mark.parametrize("wdt", [inputgen.BF16, inputgen.I8])
def test_wait_that_runs_out_is_reported_and_the_context_stays_usable(wdt):
    # int8: the fused kernel's grid-barrier counters have advanced before the error, and the
    # status call resets them; the layer must still compute correctly afterwards
    wl = inputgen.custom("fail_T1", T=1, d=256, E=8, k=2, f=256, act=inputgen.BF16, wdt=wdt)
    p = inputgen.make_problem(wl, seed=1)
    layer = H.make_layer(wl)
    H.parity(p, layer=layer)
    s = torch.cuda.Stream()
    colibri.colibri_selftest_wait_timeout(layer.ctx, 20000, stream=s)
    with pytest.raises(colibri.ColibriError) as ei:
        layer.sync_status(stream=s)
    assert ei.value.status == TIMEOUT
    layer.sync_status(stream=s)  # reported once, then cleared
    H.parity(p, layer=layer)     # the context still computes the layer correctly
    layer.sync_status()
    layer.close()


def test_selftest_rejects_bad_arguments():
    wl = inputgen.custom("fail_args", T=1, d=256, E=8, k=2, f=256)
    layer = H.make_layer(wl)
    for bad in (0, -5, 1000001):
        with pytest.raises(colibri.ColibriError) as ei:
            colibri.colibri_selftest_wait_timeout(layer.ctx, bad)
        assert ei.value.status == -1
    layer.close()
