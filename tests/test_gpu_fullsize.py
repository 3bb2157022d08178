"""Full-size parity on the benchmark's workloads (GPU vs the CPU oracle).

The benchmark's workload -- LLaMA-2-7B-shaped linears, W4A8 per-channel,
M in {1, 4, 16, 64}, 1% outlier channels x100 -- runs through qlin_forward
exactly as bench.py launches it (same entry point, same workspace layout,
stream-K decomposition over all SMs).  The oracle checks every token row for
M <= 16 and 8 sampled rows (always including the row with the largest
scale) for larger M; packed weights and codes are compared in full.
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


@pytest.mark.parametrize("wl_name,shape_idx,ms", [
    ("llama7b_w4_decode", 0, [1, 4, 16, 64]),   # q_proj 4096x4096
    ("llama7b_w4_decode", 4, [1, 16, 64]),      # gate_proj 4096->11008
    ("llama7b_w4_decode", 6, [1, 16]),          # down_proj 11008->4096
])
def test_bench_workload_sampled(q, oracle, wl_name, shape_idx, ms):
    wl = synth.WORKLOADS[wl_name]
    L0 = synth.layer(wl, shape_idx, M=1)
    W = L0["W"]
    O = L0["O"]
    layer = q.PackedLayer.pack(torch.from_numpy(W).cuda(), O, wl.fmt)
    pk = oracle.pack_layer(bits(W), O, wl.fmt)
    from layouts import tile_w4
    K, N = W.shape
    np.testing.assert_array_equal(layer.view("codes").cpu().numpy(), tile_w4(pk["packed"], N, K))
    np.testing.assert_array_equal(layer.view("chan_scale").cpu().numpy().view(np.uint32), pk["c"].view(np.uint32))
    for M in ms:
        L = synth.layer(wl, shape_idx, M=M, with_weights=False)
        X = torch.from_numpy(L["X"]).cuda()
        s = torch.ones(len(O), dtype=torch.float32, device="cuda")
        Y = torch.empty((M, L["N"]), dtype=torch.float16, device="cuda")
        nws = q.qlin_forward_workspace(M, layer.w)
        ws = q.empty_workspace(nws)
        for rep in range(2):  # the second call reuses the workspace the first left
            s.fill_(1.0)
            q.qlin_forward(X, M, layer.w, s, wl.gamma, True, Y, ws, nws)
        q.qlin_poll_device_status()
        torch.cuda.synchronize()
        r_all = oracle.forward(bits(L["X"]), bits(W), pk, np.ones(len(O), np.float32), wl.gamma,
                               rows=np.zeros(0, np.int32))
        if M <= 16:
            rows = np.arange(M, dtype=np.int32)
        else:
            rng = np.random.default_rng(M)
            rows = np.unique(np.concatenate([rng.choice(M, 7, replace=False),
                                             [int(np.argmax(r_all["a"]))]])).astype(np.int32)
        r = oracle.forward(bits(L["X"]), bits(W), pk, np.ones(len(O), np.float32), wl.gamma, rows=rows)
        np.testing.assert_array_equal(s.cpu().numpy().view(np.uint32), r["s"].view(np.uint32))
        y = Y.float().cpu().numpy().astype(np.float64)[rows]
        err = np.abs(y - r["y"]) / np.maximum(np.abs(r["y"]), 1.0)
        assert err.max() <= TOL, (M, err.max())


@pytest.mark.parametrize("fmt", [synth.W4_PERCHANNEL, synth.W4_G128, synth.W8_PERCHANNEL])
@pytest.mark.parametrize("M", [1, 16, 48])
def test_split_k_accumulators_exact(q, oracle, fmt, M):
    """Decode shapes run stream-K (tiles split over all SMs, INT32 partials
    reduced through scratch slots); the reduced accumulators are exact and
    the per-tile counters are left zeroed."""
    K, N, nO = 4096, 1024, 41
    L = synth.layer("llama7b_w4_decode", 0, M=M, K=K, N=N, n_outliers=nO)
    layer = q.PackedLayer.pack(torch.from_numpy(L["W"]).cuda(), L["O"], fmt)
    pk = oracle.pack_layer(bits(L["W"]), L["O"], fmt)
    X = torch.from_numpy(L["X"]).cuda()
    s = torch.ones(nO, dtype=torch.float32, device="cuda")
    Xq = torch.empty((M, K), dtype=torch.int8, device="cuda")
    a = torch.empty(M, dtype=torch.float32, device="cuda")
    XqO = torch.empty((M, nO), dtype=torch.int8, device="cuda")
    aws_n = q.qlin_quant_act_workspace(M, layer.w)
    aws = q.empty_workspace(aws_n)
    q.qlin_quant_act(X, M, layer.w, s, 0.9, True, Xq, a, XqO, aws, aws_n)
    gws_n = q.qlin_gemm_workspace(M, layer.w)
    gws = q.empty_workspace(gws_n)
    Y = torch.empty((M, N), dtype=torch.float16, device="cuda")
    acc = torch.empty((M, N), dtype=torch.int32, device="cuda")
    for rep in range(2):
        q.qlin_gemm(layer.w, Xq, a, XqO, s, M, Y, acc, gws, gws_n)
    q.qlin_poll_device_status()
    torch.cuda.synchronize()
    r = oracle.forward(bits(L["X"]), bits(L["W"]), pk, np.ones(nO, np.float32), 0.9)
    np.testing.assert_array_equal(acc.cpu().numpy().astype(np.int64), r["acc"])
    y = Y.float().cpu().numpy().astype(np.float64)
    err = np.abs(y - r["y"]) / np.maximum(np.abs(r["y"]), 1.0)
    assert err.max() <= TOL
    # scratch layout: [U hi/lo][INT32 partial slots][fp32 partial slots][counters];
    # partial slots are plain-overwritten, the per-tile counters must be zero again
    up = lambda v: -(-v // 256) * 256
    bt = 16 if M <= 16 else (32 if M <= 32 else 64)
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    ks = 4 if bt <= 16 else 2  # K-blocks per pipeline step for this token tile
    T = -(-(-(-K // 128)) // ks) + -(-nO // 64)
    grid = min(sms, -(-N // 128) * -(-M // bt) * T)
    u_bytes = up(2 * M * ((nO + 7) // 8 * 8) * 2)
    slots = up(2 * grid * bt * 128 * 4)
    cnt_region = gws[u_bytes + 2 * slots:u_bytes + 2 * slots + grid * 4]
    assert not cnt_region.any().item(), "stream-K counters not left zeroed"
