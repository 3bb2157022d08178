"""Grouped forwards (qlin_forward_grouped): several independent layers at
the same token count in one quantization launch and one persistent GEMM
launch.  Each problem must give exactly what its own qlin_forward gives (Y
and the momentum state bit for bit: same arithmetic, same order), and so
match the CPU oracle (s bit-exact, Y within 2e-3 * max(|y_ref|, 1)).  The
groups mix layer shapes, outlier counts (including none) and ragged
channel tiles, and the workspace is reused by a second call."""
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


def bits(a):
    return np.ascontiguousarray(a).view(np.uint16)


# (K, N, n_outlier) per problem of a group
GROUP = [(512, 256, 10), (1024, 384, 0), (768, 272, 70), (4096, 128, 9), (640, 336, 13)]


@pytest.mark.parametrize("fmt", [synth.W4_PERCHANNEL, synth.W4_G128, synth.W8_PERCHANNEL])
@pytest.mark.parametrize("M", [1, 16, 48])
def test_grouped_matches_single_and_oracle(q, oracle, fmt, M):
    probs = []
    for j, (K, N, nO) in enumerate(GROUP):
        if fmt == synth.W4_G128 and K % 128:
            continue
        L = synth.layer("small", 0, M=M, K=K, N=N, n_outliers=nO, step=j)
        L["W"] = synth.layer("small", 0, M=1, K=K, N=N, n_outliers=nO)["W"]
        layer = q.PackedLayer.pack(torch.from_numpy(L["W"]).cuda(), L["O"], fmt)
        s0 = np.random.default_rng(j).uniform(1.0, 3.0, nO).astype(np.float32)
        probs.append({"L": L, "layer": layer, "s0": s0, "K": K, "N": N, "nO": nO})
    ws_list = [p["layer"].w for p in probs]
    nws = q.qlin_forward_grouped_workspace(ws_list, M)
    wsp = q.empty_workspace(nws)
    Xs = [torch.from_numpy(p["L"]["X"]).cuda() for p in probs]
    for rep in range(2):
        ss = [torch.from_numpy(p["s0"]).cuda() if p["nO"] else torch.zeros(1, device="cuda") for p in probs]
        Ys = [torch.empty((M, p["N"]), dtype=torch.float16, device="cuda") for p in probs]
        q.qlin_forward_grouped(ws_list, Xs, ss, Ys, M, 0.9, True, wsp, nws)
        # the same problems one by one
        s1 = [torch.from_numpy(p["s0"]).cuda() if p["nO"] else torch.zeros(1, device="cuda") for p in probs]
        Y1 = [torch.empty((M, p["N"]), dtype=torch.float16, device="cuda") for p in probs]
        for p, X, s, Y in zip(probs, Xs, s1, Y1):
            n1 = q.qlin_forward_workspace(M, p["layer"].w)
            w1 = q.empty_workspace(n1)
            q.qlin_forward(X, M, p["layer"].w, s, 0.9, True, Y, w1, n1)
        q.qlin_poll_device_status()
        torch.cuda.synchronize()
        for j, p in enumerate(probs):
            tag = f"fmt={fmt} M={M} problem {j} rep {rep}"
            np.testing.assert_array_equal(Ys[j].cpu().numpy().view(np.uint16), Y1[j].cpu().numpy().view(np.uint16),
                                          err_msg=tag)
            if p["nO"]:
                np.testing.assert_array_equal(ss[j].cpu().numpy().view(np.uint32), s1[j].cpu().numpy().view(np.uint32),
                                              err_msg=tag)
            if rep == 0:
                pk = oracle.pack_layer(bits(p["L"]["W"]), p["L"]["O"], fmt)
                r = oracle.forward(bits(p["L"]["X"]), bits(p["L"]["W"]), pk, p["s0"], 0.9)
                if p["nO"]:
                    np.testing.assert_array_equal(ss[j].cpu().numpy().view(np.uint32), r["s"].view(np.uint32),
                                                  err_msg=tag)
                y = Ys[j].float().cpu().numpy().astype(np.float64)
                err = np.abs(y - r["y"]) / np.maximum(np.abs(r["y"]), 1.0)
                assert err.max() <= TOL, (tag, err.max())


def test_grouped_bench_shapes_llama70b_decode(q, oracle):
    """The 70B g128 decode bucket as the bench runs it: the four linears at
    one token in one grouped call; each Y matches qlin_forward bit for bit,
    and the oracle on q_proj and kv_proj."""
    wl = synth.WORKLOADS["llama70b_w4g128"]
    M = 1
    probs = []
    for si in range(len(wl.shapes)):
        L = synth.layer(wl, si, M=M)
        layer = q.PackedLayer.pack(torch.from_numpy(L["W"]).cuda(), L["O"], wl.fmt)
        probs.append({"L": L, "layer": layer, "N": L["N"], "nO": len(L["O"])})
    ws_list = [p["layer"].w for p in probs]
    nws = q.qlin_forward_grouped_workspace(ws_list, M)
    wsp = q.empty_workspace(nws)
    Xs = [torch.from_numpy(p["L"]["X"]).cuda() for p in probs]
    ss = [torch.ones(p["nO"], device="cuda") for p in probs]
    Ys = [torch.empty((M, p["N"]), dtype=torch.float16, device="cuda") for p in probs]
    q.qlin_forward_grouped(ws_list, Xs, ss, Ys, M, wl.gamma, True, wsp, nws)
    Y1 = []
    for p, X in zip(probs, Xs):
        s = torch.ones(p["nO"], device="cuda")
        Y = torch.empty((M, p["N"]), dtype=torch.float16, device="cuda")
        n1 = q.qlin_forward_workspace(M, p["layer"].w)
        q.qlin_forward(X, M, p["layer"].w, s, wl.gamma, True, Y, q.empty_workspace(n1), n1)
        Y1.append(Y)
    q.qlin_poll_device_status()
    torch.cuda.synchronize()
    for j in range(len(probs)):
        np.testing.assert_array_equal(Ys[j].cpu().numpy().view(np.uint16), Y1[j].cpu().numpy().view(np.uint16))
    for j in (0, 1):
        p = probs[j]
        pk = oracle.pack_layer(bits(p["L"]["W"]), p["L"]["O"], wl.fmt)
        r = oracle.forward(bits(p["L"]["X"]), bits(p["L"]["W"]), pk, np.ones(p["nO"], np.float32), wl.gamma)
        np.testing.assert_array_equal(ss[j].cpu().numpy().view(np.uint32), r["s"].view(np.uint32))
        y = Ys[j].float().cpu().numpy().astype(np.float64)
        assert (np.abs(y - r["y"]) / np.maximum(np.abs(r["y"]), 1.0)).max() <= TOL


def test_grouped_argument_errors(q):
    L = synth.layer("small", 0, M=4, K=512, N=128, n_outliers=3)
    a = q.PackedLayer.pack(torch.from_numpy(L["W"]).cuda(), L["O"], synth.W4_PERCHANNEL)
    b = q.PackedLayer.pack(torch.from_numpy(L["W"]).cuda(), L["O"], synth.W8_PERCHANNEL)
    with pytest.raises(q.QlinError) as e:
        q.qlin_forward_grouped_workspace([a.w] * 33, 4)
    assert q.STATUS[e.value.status] == "QLIN_ERR_SHAPE"
    with pytest.raises(q.QlinError) as e:
        q.qlin_forward_grouped_workspace([a.w], 65)
    assert q.STATUS[e.value.status] == "QLIN_ERR_SHAPE"
    with pytest.raises(q.QlinError) as e:
        q.qlin_forward_grouped_workspace([a.w, b.w], 4)
    assert q.STATUS[e.value.status] == "QLIN_ERR_ARG"
    X = torch.from_numpy(L["X"]).cuda()
    s = torch.ones(3, device="cuda")
    Y = torch.empty((4, 128), dtype=torch.float16, device="cuda")
    n = q.qlin_forward_grouped_workspace([a.w, a.w], 4)
    with pytest.raises(q.QlinError) as e:  # the same output twice
        q.qlin_forward_grouped([a.w, a.w], [X, X], [s, s], [Y, Y], 4, 0.9, True, q.empty_workspace(n), n)
    assert q.STATUS[e.value.status] == "QLIN_ERR_ARG"
