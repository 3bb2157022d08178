"""GPU parity: the CUDA library (through its C ABI) against the CPU oracle.

Bit-exact: packed codes and scales, W_O^T, wmax_O, activation codes, token
scales, the outlier codes, the momentum state and the INT32 accumulators.
FP16 outputs: |y - y_ref| <= 2e-3 * max(|y_ref|, 1) against the oracle's
fp64 dequant (the tolerance the layer is specified to).
"""
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


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def case(fmt, M, K, N, nO, seed_shape=0, wl="small"):
    L = synth.layer(wl, seed_shape, M=M, K=K, N=N, n_outliers=nO)
    L["fmt"] = fmt
    return L


def run_gpu(q, L, s0, gamma, update=True, with_forward=True):
    fmt, M, K, N = L["fmt"], L["M"], L["K"], L["N"]
    O = L["O"]
    nO = len(O)
    Wd = dev(L["W"])
    layer = q.PackedLayer.pack(Wd, O, fmt)
    Xd = dev(L["X"])
    s = dev(s0.astype(np.float32)) if nO else torch.zeros(1, device="cuda")
    Xq = torch.empty((M, K), dtype=torch.int8, device="cuda")
    a = torch.empty(M, dtype=torch.float32, device="cuda")
    XqO = torch.empty((M, max(nO, 1)), dtype=torch.int8, device="cuda")
    aws_n = q.qlin_quant_act_workspace(M, layer.w)
    aws = q.empty_workspace(aws_n)
    q.qlin_quant_act(Xd, M, layer.w, s, gamma, update, Xq, a, XqO, aws, aws_n)
    Y = torch.empty((M, N), dtype=torch.float16, device="cuda")
    acc = torch.empty((M, N), dtype=torch.int32, device="cuda")
    gws_n = q.qlin_gemm_workspace(M, layer.w)
    gws = q.empty_workspace(gws_n)
    q.qlin_gemm(layer.w, Xq, a, XqO, s, M, Y, acc, gws, gws_n)
    out = {"layer": layer, "Xq": Xq, "a": a, "XqO": XqO[:, :nO], "s": s[:nO], "Y": Y, "acc": acc,
           "aws": aws}
    if with_forward:
        s2 = dev(s0.astype(np.float32)) if nO else torch.zeros(1, device="cuda")
        Y2 = torch.empty((M, N), dtype=torch.float16, device="cuda")
        fws_n = q.qlin_forward_workspace(M, layer.w)
        fws = q.empty_workspace(fws_n)
        q.qlin_forward(Xd, M, layer.w, s2, gamma, update, Y2, fws, fws_n)
        out["Y_fwd"] = Y2
        out["s_fwd"] = s2[:nO]
    q.qlin_poll_device_status()
    torch.cuda.synchronize()
    return out


def check_pack(oracle, L, g):
    from layouts import tile_w4, tile_w8, tile_wot
    fmt = L["fmt"]
    K, N = L["W"].shape
    pk = oracle.pack_layer(bits(L["W"]), L["O"], fmt)
    layer = g["layer"]
    want = tile_w8(pk["packed"], N, K) if fmt == synth.W8_PERCHANNEL else tile_w4(pk["packed"], N, K)
    np.testing.assert_array_equal(layer.view("codes").cpu().numpy(), want)
    np.testing.assert_array_equal(layer.view("chan_scale").cpu().numpy().view(np.uint32), pk["c"].view(np.uint32))
    if fmt == synth.W4_G128:
        np.testing.assert_array_equal(layer.view("group_scale").cpu().numpy().view(np.uint16), pk["g_h"])
        np.testing.assert_array_equal(layer.view("fold_ratio").cpu().numpy().view(np.uint16), pk["r_h"])
    nO = len(L["O"])
    if nO:
        wot = layer.view("W_Ot").cpu().numpy().view(np.uint16)
        np.testing.assert_array_equal(wot, tile_wot(bits(L["W"])[L["O"], :].T, N, nO))
        np.testing.assert_array_equal(layer.view("wmax_O").cpu().numpy().view(np.uint32),
                                      pk["wmaxO"].view(np.uint32))
        np.testing.assert_array_equal(layer.view("outlier_idx").cpu().numpy(), L["O"])
    return pk


def check_all(oracle, L, g, s0, gamma, update=True):
    pk = check_pack(oracle, L, g)
    r = oracle.forward(bits(L["X"]), bits(L["W"]), pk, s0, gamma, update_momentum=update)
    nO = len(L["O"])
    if nO:
        np.testing.assert_array_equal(g["s"].cpu().numpy().view(np.uint32), r["s"].view(np.uint32))
    np.testing.assert_array_equal(g["Xq"].cpu().numpy(), r["Xq"])
    np.testing.assert_array_equal(g["a"].cpu().numpy().view(np.uint32), r["a"].view(np.uint32))
    if nO:
        np.testing.assert_array_equal(g["XqO"].cpu().numpy(), r["XqO"])
    np.testing.assert_array_equal(g["acc"].cpu().numpy().astype(np.int64), r["acc"])
    y = g["Y"].float().cpu().numpy().astype(np.float64)
    err = np.abs(y - r["y"]) / np.maximum(np.abs(r["y"]), 1.0)
    assert err.max() <= TOL, f"max scaled error {err.max():.3e}"
    if "Y_fwd" in g:
        # the fused path computes the same values in the same order
        np.testing.assert_array_equal(g["Y_fwd"].cpu().numpy().view(np.uint16), g["Y"].cpu().numpy().view(np.uint16))
        if nO:
            np.testing.assert_array_equal(g["s_fwd"].cpu().numpy().view(np.uint32), r["s"].view(np.uint32))
    if nO and update:
        # the act-quant scratch is left zero for the next call
        assert not g["aws"].any().item()
    return r


FMTS = [synth.W4_PERCHANNEL, synth.W4_G128, synth.W8_PERCHANNEL]


@pytest.mark.parametrize("fmt", FMTS)
def test_small_workload(q, oracle, fmt):
    L = synth.layer("small", 0)
    L["fmt"] = fmt
    s0 = np.ones(len(L["O"]), np.float32)
    g = run_gpu(q, L, s0, L["gamma"])
    check_all(oracle, L, g, s0, L["gamma"])


SHAPE_MKN = [
    (1, 512, 256, 10),      # single token (decode), BT = 16
    (4, 1024, 128, 3),
    (16, 640, 336, 13),     # ragged N tile, n_outlier not a multiple of 8
    (37, 768, 272, 70),     # ragged M, two compensation K-steps
    (64, 2048, 384, 0),     # no outliers: the plain QQQ path
    (200, 1152, 256, 41),   # BT = 256 with a ragged token tile
    (130, 4096, 128, 9),    # 32 K-steps: the stage ring wraps several times
    (700, 512, 384, 17),    # 3 x 3 tiles of 256 tokens: token-tile-fastest raster order, ragged last token tile
]
SHAPES = [(fmt, *mknO) for fmt in FMTS for mknO in SHAPE_MKN]


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("M,K,N,nO", SHAPE_MKN)
def test_shapes(q, oracle, fmt, M, K, N, nO):
    L = case(fmt, M, K, N, nO, seed_shape=0)
    rng = np.random.default_rng(M * 7 + K)
    s0 = rng.uniform(1.0, 4.0, nO).astype(np.float32)
    g = run_gpu(q, L, s0, 0.9)
    check_all(oracle, L, g, s0, 0.9)


@pytest.mark.parametrize("fmt", FMTS)
def test_maximum_k_and_outliers(q, oracle, fmt):
    # the largest supported layer depth with the largest outlier set: the
    # quantization row (128 KiB) and outlier tables fill the shared memory,
    # 512 K-blocks stream through the rings, 64 compensation slices
    L = case(fmt, 3, 65536, 128, 4096)
    rng = np.random.default_rng(65536)
    s0 = rng.uniform(1.0, 3.0, 4096).astype(np.float32)
    g = run_gpu(q, L, s0, 0.9)
    check_all(oracle, L, g, s0, 0.9)


@pytest.mark.parametrize("fmt", [synth.W4_PERCHANNEL, synth.W8_PERCHANNEL])
def test_ragged_k(q, oracle, fmt):
    # K a multiple of 32 but not of 128: the last K-step is zero-filled by TMA
    L = case(fmt, 23, 608, 144, 5)
    s0 = np.ones(5, np.float32)
    g = run_gpu(q, L, s0, 0.5)
    check_all(oracle, L, g, s0, 0.5)


def test_no_momentum_update(q, oracle):
    L = case(synth.W4_PERCHANNEL, 16, 512, 256, 12)
    s0 = np.random.default_rng(3).uniform(1.0, 9.0, 12).astype(np.float32)
    g = run_gpu(q, L, s0, 0.9, update=False)
    check_all(oracle, L, g, s0, 0.9, update=False)


def test_zero_token_and_zero_channel(q, oracle):
    L = case(synth.W4_G128, 16, 512, 128, 6)
    L["X"][3] = 0
    L["W"][:, 17] = 0
    L["W"][128:256, 40] = 0  # one all-zero group
    s0 = np.ones(6, np.float32)
    g = run_gpu(q, L, s0, 0.9)
    check_all(oracle, L, g, s0, 0.9)
    assert g["a"][3].item() == 0.0


def test_quaff_momentum_steps(q, oracle):
    """Quaff W8A8 forward over several steps with drifting outlier magnitudes
    (the Phi-3 workload's recipe at a reduced size): s, codes and INT32 stay
    bit-exact at every step."""
    wl = synth.WORKLOADS["phi3_w8_quaff"]
    K, N, M = 1024, 256, 64
    nO = 80
    L0 = synth.layer(wl, 3, M=M, K=K, N=N, n_outliers=nO, step=0)
    Wd = dev(L0["W"])
    layer = q.PackedLayer.pack(Wd, L0["O"], synth.W8_PERCHANNEL)
    pk = oracle.pack_layer(bits(L0["W"]), L0["O"], synth.W8_PERCHANNEL)
    s_dev = torch.ones(nO, dtype=torch.float32, device="cuda")
    s_ref = np.ones(nO, np.float32)
    fws_n = q.qlin_forward_workspace(M, layer.w)
    fws = q.empty_workspace(fws_n)
    Y = torch.empty((M, N), dtype=torch.float16, device="cuda")
    for step in range(8):
        L = synth.layer(wl, 3, M=M, K=K, N=N, n_outliers=nO, step=step, with_weights=False)
        q.qlin_forward(dev(L["X"]), M, layer.w, s_dev, wl.gamma, True, Y, fws, fws_n)
        r = oracle.forward(bits(L["X"]), bits(L0["W"]), pk, s_ref, wl.gamma)
        s_ref = r["s"]
        torch.cuda.synchronize()
        np.testing.assert_array_equal(s_dev.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))
        y = Y.float().cpu().numpy().astype(np.float64)
        err = np.abs(y - r["y"]) / np.maximum(np.abs(r["y"]), 1.0)
        assert err.max() <= TOL, (step, err.max())
    q.qlin_poll_device_status()


def test_data_parallel_split_matches_fused(q, oracle):
    """colmax -> (external MAX reduce) -> momentum update -> quant(update=0)
    gives the same s and codes as the fused update."""
    L = case(synth.W4_PERCHANNEL, 48, 512, 128, 11)
    nO = 11
    layer = q.PackedLayer.pack(dev(L["W"]), L["O"], synth.W4_PERCHANNEL)
    X = dev(L["X"])
    halves = [X[:20], X[20:]]
    cm = [torch.empty(nO, dtype=torch.float32, device="cuda") for _ in halves]
    for h, c in zip(halves, cm):
        q.qlin_outlier_colmax(h, h.shape[0], layer.w, c)
    cmax = torch.maximum(cm[0], cm[1])
    s = torch.ones(nO, dtype=torch.float32, device="cuda")
    q.qlin_momentum_update(layer.w, cmax, s, 0.9)
    pk = oracle.pack_layer(bits(L["W"]), L["O"], synth.W4_PERCHANNEL)
    s_ref = oracle.momentum_update(bits(L["X"]), L["O"], pk["wmaxO"], 0.9, np.ones(nO, np.float32))
    torch.cuda.synchronize()
    np.testing.assert_array_equal(s.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))


def test_zero_tokens_is_noop(q):
    L = case(synth.W8_PERCHANNEL, 4, 256, 128, 3)
    layer = q.PackedLayer.pack(dev(L["W"]), L["O"], synth.W8_PERCHANNEL)
    q.qlin_gemm(layer.w, None, None, None, None, 0, None, None, None, 0)
    q.qlin_forward(None, 0, layer.w, None, 0.9, True, None, None, 0)
    q.qlin_poll_device_status()
