"""Failures inside a kernel reach the caller through the sticky status word.

A kernel that cannot finish (here: a bounded wait that runs out) must not
hang the GPU or fault, and must not let the call look successful.  The test
hook LUTGEMM_TEST_STALL makes every warp of the lookup kernel wait for a
barrier that nothing signals; the wait gives up after 1 ms, the warp lets its
copies in flight land, stops, and sets LUTGEMM_STATUS_TIMEOUT.  These tests
check that the bit is reported (and raised by the binding's ``check``), that
clearing works, and that the context and the workspace are fit for the next
call, whose result must match the oracle.
"""
from __future__ import annotations

import pytest
import torch

import bcq_synth as S
from oracle import bcq_oracle as O
from tests._tol import compare

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module")
def L():
    from weight_only_quantized_bcq_b200 import lutgemm
    lutgemm.lib()
    assert torch.cuda.is_available()
    return lutgemm


def _problem(q, m, n, g, batch, seed):
    gen = S.generator(seed)
    signs = S.draw_signs(gen, q, m, n)
    alpha = S.draw_alpha(gen, q, m, n, g, 0.02)
    x = S.draw_x(gen, batch, n)
    return signs, alpha, x


# (one slice: y written by the lookup kernel), (contiguous unit ranges),
# (per-segment groups with counter tiles)
SHAPES = [(3, 512, 512, 128, 1), (3, 64, 1024, 128, 200), (3, 2048, 4096, 128, 37)]


@pytest.mark.parametrize("q,m,n,g,batch", SHAPES)
def test_stalled_run_reports_timeout_then_recovers(L, q, m, n, g, batch):
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    signs, alpha, x = _problem(q, m, n, g, batch, 60 + batch)
    packed = L.pack_bcq(signs.to(DEV))
    a_d, x_d = alpha.to(DEV), x.to(DEV)
    ws = L.new_workspace(m, n, batch, q, g)
    L.run(packed, a_d, x_d, m, n, q, g, workspace=ws, _flags=L.TEST_STALL)
    assert L.workspace_status(ws, clear=False) == L.STATUS_TIMEOUT
    assert L.workspace_status(ws, clear=True) == L.STATUS_TIMEOUT
    assert L.workspace_status(ws, clear=False) == 0
    # The counters were reset by the stalled call too.
    assert not ws[256: 256 + 4096].cpu().numpy().any()
    # The binding's check raises on a stalled call.
    with pytest.raises(L.LutgemmDeviceError) as e:
        L.run(packed, a_d, x_d, m, n, q, g, workspace=ws, check=True, _flags=L.TEST_STALL)
    assert e.value.bits == L.STATUS_TIMEOUT
    assert L.workspace_status(ws) == 0          # check cleared it
    # The next call on the same workspace is correct and reports nothing.
    y = L.run(packed, a_d, x_d, m, n, q, g, workspace=ws, check=True)
    y_ref = O.bcq_matmul(x.numpy(), signs.numpy(), alpha.numpy(), g)
    ok, st = compare(y.cpu().numpy(), y_ref, alpha.numpy(), x.numpy(), n)
    assert ok, (st, L.launch_plan(m, n, batch, sms))


def test_status_stays_zero_over_many_normal_runs(L):
    q, m, n, g, batch = 3, 1000, 6144, 128, 3
    signs, alpha, x = _problem(q, m, n, g, batch, 5)
    packed = L.pack_bcq(signs.to(DEV))
    ws = L.new_workspace(m, n, batch, q, g)
    for _ in range(20):
        L.run(packed, alpha.to(DEV), x.to(DEV), m, n, q, g, workspace=ws)
    assert L.workspace_status(ws) == 0


def test_tensor_core_calls_report_through_their_words(L):
    """lutgemm_run_tc uses the library's word; lutgemm_run's tensor-core
    dispatch uses the workspace's.  Normal runs leave both at zero."""
    q, m, n, g, batch = 3, 256, 2048, 128, 40
    signs, alpha, x = _problem(q, m, n, g, batch, 8)
    packed = L.pack_bcq(signs.to(DEV))
    L.library_status(clear=True)
    y = L.run_tc(packed, alpha.to(DEV), x.to(DEV), m, n, q, g, check=True)
    ws = L.new_workspace(m, n, batch, q, g)
    y2 = L.run(packed, alpha.to(DEV), x.to(DEV), m, n, q, g, workspace=ws, allow_tensor_cores=True)
    assert L.workspace_status(ws) == 0 and L.library_status() == 0
    y_ref = O.bcq_matmul(x.numpy(), signs.numpy(), alpha.numpy(), g)
    for out in (y, y2):
        ok, st = compare(out.cpu().numpy(), y_ref, alpha.numpy(), x.numpy(), n)
        assert ok, st
