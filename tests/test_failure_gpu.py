"""Failure detection without a GPU fault: the library's bounded device waits
are made to expire on purpose (an mbarrier that nothing arrives on; a grid
barrier missing one CTA's arrival, suppressed by a host-set parameter).  The
expiry must surface as MOE_ERR_TIMEOUT in the workspace error word, the
kernel must end within a bounded multiple of the wait limit, and the context
must stay usable: a layer computed afterwards still matches the oracle."""
import pytest

import gen
from gpu_util import check_output, check_routing, run_layer

pytestmark = pytest.mark.gpu

LIMIT_NS = 2_000_000          # each wait gives up after 2 ms


def _timed_selftest(m, ws, kind, ctas, skip):
    import torch
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record()
    m.moe_wait_selftest(kind, ctas, skip, LIMIT_NS, ws)
    end.record()
    err = m.moe_get_device_error(ws)      # synchronises the stream
    return err, start.elapsed_time(end)


@pytest.mark.parametrize("kind,ctas,skip", [(0, 1, -1), (1, 8, 3), (1, 148, 0), (1, 148, 147)])
def test_expired_wait_reports_timeout(kind, ctas, skip):
    import torch
    import bit_dequant_expert_b200 as m
    ws = torch.zeros(4096, dtype=torch.uint8, device="cuda")
    m.moe_workspace_init(ws)
    err, ms = _timed_selftest(m, ws, kind, ctas, skip)
    assert err == m.MOE_ERR_TIMEOUT
    # the waits lasted about the limit, and ended
    assert 0.5 * LIMIT_NS / 1e6 <= ms < 1000.0
    # the error word is sticky until the workspace is re-initialised
    assert m.moe_get_device_error(ws) == m.MOE_ERR_TIMEOUT
    m.moe_workspace_init(ws)
    assert m.moe_get_device_error(ws) == 0


def test_complete_barrier_reports_nothing():
    import torch
    import bit_dequant_expert_b200 as m
    ws = torch.zeros(4096, dtype=torch.uint8, device="cuda")
    m.moe_workspace_init(ws)
    _timed_selftest(m, ws, 1, 148, -1)     # first launch loads the kernel; not timed
    for _ in range(3):
        err, ms = _timed_selftest(m, ws, 1, 148, -1)
        assert err == 0
        assert ms < 0.5 * LIMIT_NS / 1e6


def test_context_usable_after_expired_waits():
    import torch
    import bit_dequant_expert_b200 as m
    ws = torch.zeros(4096, dtype=torch.uint8, device="cuda")
    m.moe_workspace_init(ws)
    m.moe_wait_selftest(0, 1, -1, LIMIT_NS, ws)
    m.moe_wait_selftest(1, 148, 5, LIMIT_NS, ws)
    assert m.moe_get_device_error(ws) == m.MOE_ERR_TIMEOUT
    # a whole layer afterwards, on another workspace: the fused decode layer and the four calls
    for T in (8, 33):
        lay = gen.make_layer(gen.config(0).with_T(T))
        out, _ = run_layer(lay, m.MOE_MODE_SCATTER, m.MOE_PATH_AUTO)
        assert out["err"] == 0
        check_routing(out, lay)
        check_output(out, lay, list(range(T)))
