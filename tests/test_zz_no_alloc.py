"""The allocation-free quantization entry point (qlin_quant_act_noalloc).

Some callers cannot allocate device memory -- a plugin inside a host
framework that owns every GPU buffer, or a latency-bound loop that must not
call cudaMalloc -- so they cannot provide qlin_quant_act's workspace.  The
no-alloc variant keeps that scratch in a fixed array inside the library.
This file checks it through the C ABI against qlin_quant_act (with a
workspace) and against the CPU oracle's momentum update and quantization,
on two calls in a row, which also exercises the scratch being reused after
the first call left it.  Collected last on purpose.
"""
import numpy as np
import pytest
import torch

from quantized_linear_layers_token_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def q():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from quantized_linear_layers_token_b200 import qlin
    qlin.lib()
    return qlin


@pytest.mark.parametrize("fmt,M,K,N,nO", [
    (synth.W4_PERCHANNEL, 16, 512, 256, 10),
    (synth.W8_PERCHANNEL, 67, 1024, 128, 77),
])
def test_noalloc_matches_workspace_path_twice(q, oracle, fmt, M, K, N, nO):
    L0 = synth.layer("small", 0, M=M, K=K, N=N, n_outliers=nO)
    wmaxO = oracle.outlier_wmax(np.ascontiguousarray(L0["W"]).view(np.uint16), L0["O"])
    s_oracle = np.ones(nO, np.float32)
    layer = q.PackedLayer.pack(torch.from_numpy(L0["W"]).cuda(), L0["O"], fmt)
    s_ref = torch.ones(nO, dtype=torch.float32, device="cuda")
    s_new = torch.ones(nO, dtype=torch.float32, device="cuda")
    nws = q.qlin_quant_act_workspace(M, layer.w)
    ws = q.empty_workspace(nws)
    for step in range(2):
        L = synth.layer("small", 0, M=M, K=K, N=N, n_outliers=nO, step=step, with_weights=False)
        if step:  # a different batch on the second call
            L["X"] = (L["X"].astype(np.float32) * np.float32(0.7)).astype(np.float16)
        X = torch.from_numpy(L["X"]).cuda()
        outs = []
        for fn, s in [("ws", s_ref), ("noalloc", s_new)]:
            Xq = torch.empty((M, K), dtype=torch.int8, device="cuda")
            a = torch.empty(M, dtype=torch.float32, device="cuda")
            XqO = torch.empty((M, nO), dtype=torch.int8, device="cuda")
            if fn == "ws":
                q.qlin_quant_act(X, M, layer.w, s, 0.9, True, Xq, a, XqO, ws, nws)
            else:
                q.qlin_quant_act_noalloc(X, M, layer.w, s, 0.9, True, Xq, a, XqO)
            outs.append((Xq, a, XqO))
        q.qlin_poll_device_status()
        torch.cuda.synchronize()
        # both paths run the same kernels: results agree exactly
        assert torch.equal(s_ref.view(torch.int32), s_new.view(torch.int32)), step
        for x, y in zip(outs[0], outs[1]):
            assert torch.equal(x.view(torch.uint8) if x.dtype == torch.int8 else x.view(torch.int32),
                               y.view(torch.uint8) if y.dtype == torch.int8 else y.view(torch.int32)), step
        assert (s_new > 1.0).all()
        # and both equal the oracle, bit for bit
        Xb = np.ascontiguousarray(L["X"]).view(np.uint16)
        s_oracle = oracle.momentum_update(Xb, L0["O"], wmaxO, 0.9, s_oracle)
        Xq_r, a_r, XqO_r = oracle.quant_act(Xb, L0["O"], s_oracle)
        np.testing.assert_array_equal(s_new.cpu().numpy().view(np.uint32), s_oracle.view(np.uint32))
        np.testing.assert_array_equal(outs[1][0].cpu().numpy(), Xq_r)
        np.testing.assert_array_equal(outs[1][1].cpu().numpy().view(np.uint32), a_r.view(np.uint32))
        np.testing.assert_array_equal(outs[1][2].cpu().numpy(), XqO_r)


def test_noalloc_rejects_too_many_outliers(q):
    K, N, nO, M = 2048, 128, 1025, 4
    layer = q.PackedLayer(K, N, synth.W8_PERCHANNEL, nO)
    X = torch.zeros((M, K), dtype=torch.float16, device="cuda")
    s = torch.ones(nO, dtype=torch.float32, device="cuda")
    Xq = torch.empty((M, K), dtype=torch.int8, device="cuda")
    a = torch.empty(M, dtype=torch.float32, device="cuda")
    XqO = torch.empty((M, nO), dtype=torch.int8, device="cuda")
    with pytest.raises(q.QlinError) as e:
        q.qlin_quant_act_noalloc(X, M, layer.w, s, 0.9, True, Xq, a, XqO)
    assert q.STATUS[e.value.status] == "QLIN_ERR_SHAPE"
    assert "1024" in str(e.value)
