"""Failure detection: every pipeline wait of the GEMM is bounded.  With the
wait limit set to zero (the library's test knob) the first wait that is not
already complete gives up; the kernel sets the device error word, drains
its copies and tensor-core work and frees its tensor memory, and
qlin_poll_device_status reports QLIN_ERR_TIMEOUT.  Afterwards, with the
default limit back, a normal forward on a zero-filled workspace matches the
oracle: the context and the library recovered.  No fault is provoked: the
wait runs out on data that would have arrived.  The layer is sized, and
the GEMM held to one persistent CTA, so that a wait is certainly pending
when it is first tested."""
import numpy as np
import pytest
import torch

from quantized_linear_layers_token_b200 import synth

pytestmark = pytest.mark.gpu
TOL = 2e-3


@pytest.fixture(scope="module")
def q():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from quantized_linear_layers_token_b200 import qlin
    qlin.lib()
    return qlin


def test_zero_wait_limit_reports_timeout_then_recovers(q, oracle):
    # one persistent CTA walks a long K loop, so its pipeline waits cannot all
    # be complete at their first test (a short loop can finish inside it)
    L = synth.layer("small", 0, M=16, K=16384, N=256, n_outliers=10)
    M, K, N, O = L["M"], L["K"], L["N"], L["O"]
    layer = q.PackedLayer.pack(torch.from_numpy(L["W"]).cuda(), O, synth.W4_PERCHANNEL)
    X = torch.from_numpy(L["X"]).cuda()
    Y = torch.empty((M, N), dtype=torch.float16, device="cuda")
    n = q.qlin_forward_workspace(M, layer.w)
    ws = q.empty_workspace(n)
    s = torch.ones(len(O), dtype=torch.float32, device="cuda")
    q.qlin_poll_device_status()  # nothing pending
    with q.knobs(wait_ns=0, cluster=0, max_ctas=1):
        q.qlin_forward(X, M, layer.w, s, L["gamma"], True, Y, ws, n)
        with pytest.raises(q.QlinError) as e:
            q.qlin_poll_device_status()
    assert q.STATUS[e.value.status] == "QLIN_ERR_TIMEOUT"
    assert q.qlin_debug_get(q.QLIN_KNOB_WAIT_NS) == 2_000_000_000
    q.qlin_poll_device_status()  # the error word was cleared
    # recovery: zero-filled workspace, fresh state, default limit
    ws.zero_()
    s.fill_(1.0)
    q.qlin_forward(X, M, layer.w, s, L["gamma"], True, Y, ws, n)
    q.qlin_poll_device_status()
    torch.cuda.synchronize()
    Wb = np.ascontiguousarray(L["W"]).view(np.uint16)
    pk = oracle.pack_layer(Wb, O, synth.W4_PERCHANNEL)
    r = oracle.forward(np.ascontiguousarray(L["X"]).view(np.uint16), Wb, pk, np.ones(len(O), np.float32), L["gamma"])
    np.testing.assert_array_equal(s.cpu().numpy().view(np.uint32), r["s"].view(np.uint32))
    y = Y.float().cpu().numpy().astype(np.float64)
    assert (np.abs(y - r["y"]) / np.maximum(np.abs(r["y"]), 1.0)).max() <= TOL
