"""Full-size parity on the benchmark's workloads (GPU vs the CPU oracle).

Every workload the benchmark measures runs here at its full size, through
the same entry points and launch configuration bench.py times:
  - LLaMA-2-7B-shaped linears, W4A8 per-channel, decode M in {1, 4, 16, 64};
  - the same linears, W4A8 g128, prefill M up to 4096 (INT4 widened once per
    call, then the INT8 kernel with 256-token tiles);
  - LLaMA-2-70B-shaped linears, W4A8 g128, M in {1, 16, 128, 1024, 8192},
    the largest K (28672) and the largest N (28672);
  - the Phi-3-mini W8A8 workload over its 20 momentum steps at M = 4096.
Packed weights, the momentum state and the activation codes Xq, a and XqO
are compared in full and bit for bit; the INT32 accumulators bit for bit on
every row up to 64 tokens, else on 16 seeded rows plus the row of largest
scale (the single-threaded oracle GEMM costs up to ~0.2 s per row here); Y
within 2e-3 * max(|y_ref|, 1) on those rows.
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


def check_packed(layer, pk, fmt, K, N):
    from layouts import tile_w4, tile_w8
    want = tile_w8(pk["packed"], N, K) if fmt == synth.W8_PERCHANNEL else tile_w4(pk["packed"], N, K)
    np.testing.assert_array_equal(layer.view("codes").cpu().numpy(), want)
    np.testing.assert_array_equal(layer.view("chan_scale").cpu().numpy().view(np.uint32), pk["c"].view(np.uint32))
    if fmt == synth.W4_G128:
        np.testing.assert_array_equal(layer.view("fold_ratio").cpu().numpy().view(np.uint16), pk["r_h"])
        np.testing.assert_array_equal(layer.view("group_scale").cpu().numpy().view(np.uint16), pk["g_h"])
    if len(pk["O"]):
        np.testing.assert_array_equal(layer.view("wmax_O").cpu().numpy().view(np.uint32),
                                      pk["wmaxO"].view(np.uint32))


def sampled_rows(M, a_gpu, seed):
    """Every row up to 64 tokens; else 16 seeded rows and the row of
    largest scale."""
    if M <= 64:
        return np.arange(M, dtype=np.int32)
    rng = np.random.default_rng(seed)
    return np.unique(np.concatenate([rng.choice(M, 16, replace=False), [int(np.argmax(a_gpu))]])).astype(np.int32)


def run_full_forward(q, oracle, wl, shape_idx, ms):
    """The bench's forward of one linear at each token count, checked
    against the oracle: qlin_forward (as timed), then qlin_quant_act +
    qlin_gemm with the INT32 accumulators exported, which must give the
    same Y bit for bit."""
    L0 = synth.layer(wl, shape_idx, M=1)
    W, O = L0["W"], L0["O"]
    K, N = W.shape
    nO = len(O)
    layer = q.PackedLayer.pack(torch.from_numpy(W).cuda(), O, wl.fmt)
    pk = oracle.pack_layer(bits(W), O, wl.fmt)
    check_packed(layer, pk, wl.fmt, K, N)
    for M in ms:
        L = synth.layer(wl, shape_idx, M=M, with_weights=False)
        X = torch.from_numpy(L["X"]).cuda()
        s = torch.ones(max(nO, 1), dtype=torch.float32, device="cuda")
        Y = torch.empty((M, N), dtype=torch.float16, device="cuda")
        nws = q.qlin_forward_workspace(M, layer.w)
        ws = q.empty_workspace(nws)
        for rep in range(2):  # the second call reuses the workspace the first left
            s.fill_(1.0)
            q.qlin_forward(X, M, layer.w, s, wl.gamma, True, Y, ws, nws)
        s2 = torch.ones(max(nO, 1), dtype=torch.float32, device="cuda")
        Xq = torch.empty((M, K), dtype=torch.int8, device="cuda")
        a = torch.empty(M, dtype=torch.float32, device="cuda")
        XqO = torch.empty((M, max(nO, 1)), dtype=torch.int8, device="cuda")
        aws_n = q.qlin_quant_act_workspace(M, layer.w)
        aws = q.empty_workspace(aws_n)
        q.qlin_quant_act(X, M, layer.w, s2, wl.gamma, True, Xq, a, XqO, aws, aws_n)
        gws_n = q.qlin_gemm_workspace(M, layer.w)
        gws = q.empty_workspace(gws_n)
        Y2 = torch.empty((M, N), dtype=torch.float16, device="cuda")
        acc = torch.empty((M, N), dtype=torch.int32, device="cuda")
        q.qlin_gemm(layer.w, Xq, a, XqO, s2, M, Y2, acc, gws, gws_n)
        q.qlin_poll_device_status()
        torch.cuda.synchronize()
        a_gpu = a.cpu().numpy()
        rows = sampled_rows(M, a_gpu, seed=M + 31 * shape_idx)
        r = oracle.forward(bits(L["X"]), bits(W), pk, np.ones(nO, np.float32), wl.gamma, rows=rows)
        tag = f"{wl.name} {L['name']} M={M}"
        if nO:
            np.testing.assert_array_equal(s.cpu().numpy()[:nO].view(np.uint32), r["s"].view(np.uint32), err_msg=tag)
            np.testing.assert_array_equal(s2.cpu().numpy()[:nO].view(np.uint32), r["s"].view(np.uint32), err_msg=tag)
            np.testing.assert_array_equal(XqO.cpu().numpy()[:, :nO], r["XqO"], err_msg=tag)
        np.testing.assert_array_equal(Xq.cpu().numpy(), r["Xq"], err_msg=tag)
        np.testing.assert_array_equal(a_gpu.view(np.uint32), r["a"].view(np.uint32), err_msg=tag)
        np.testing.assert_array_equal(acc.cpu().numpy()[rows].astype(np.int64), r["acc"], err_msg=tag)
        np.testing.assert_array_equal(Y.cpu().numpy().view(np.uint16), Y2.cpu().numpy().view(np.uint16), err_msg=tag)
        y = Y.float().cpu().numpy().astype(np.float64)[rows]
        err = np.abs(y - r["y"]) / np.maximum(np.abs(r["y"]), 1.0)
        assert err.max() <= TOL, (tag, err.max())
        del X, Y, Y2, acc, Xq, ws, gws
        torch.cuda.empty_cache()


@pytest.mark.parametrize("wl_name,shape_idx,ms", [
    ("llama7b_w4_decode", 0, [1, 4, 16, 64]),   # q_proj 4096x4096
    ("llama7b_w4_decode", 4, [1, 16, 64]),      # gate_proj 4096->11008
    ("llama7b_w4_decode", 6, [1, 4, 16, 64]),   # down_proj 11008->4096
])
def test_bench_workload_sampled(q, oracle, wl_name, shape_idx, ms):
    run_full_forward(q, oracle, synth.WORKLOADS[wl_name], shape_idx, ms)


@pytest.mark.parametrize("shape_idx,ms", [
    (4, [512, 4096]),   # gate_proj 4096->11008
    (6, [2048, 4096]),  # down_proj 11008->4096
])
def test_llama7b_g128_prefill_full_size(q, oracle, shape_idx, ms):
    run_full_forward(q, oracle, synth.WORKLOADS["llama7b_w4g128_prefill"], shape_idx, ms)


@pytest.mark.parametrize("shape_idx", [2, 3])  # up_proj 8192->28672, down_proj 28672->8192
def test_llama70b_g128_full_size(q, oracle, shape_idx):
    run_full_forward(q, oracle, synth.WORKLOADS["llama70b_w4g128"], shape_idx, [1, 16, 128, 1024, 8192])


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


def test_phi3_quaff_twenty_steps(q, oracle):
    """The Phi-3-mini W8A8 workload as specified: qkv_proj at M = 4096 over
    20 steps, outlier magnitudes drifting and X redrawn each step, the
    momentum state carried from step to step.  Every step: s bit-exact, the
    codes Xq, a and XqO in full, INT32 accumulators exact on 16 seeded rows
    and the row of largest scale (the single-threaded oracle GEMM takes
    ~0.2 s per row at this shape), Y within the tolerance there."""
    wl = synth.WORKLOADS["phi3_w8_quaff"]
    si = 0
    L0 = synth.layer(wl, si, M=1)
    W, O = L0["W"], L0["O"]
    K, N = W.shape
    M, nO = 4096, len(O)
    layer = q.PackedLayer.pack(torch.from_numpy(W).cuda(), O, wl.fmt)
    pk = oracle.pack_layer(bits(W), O, wl.fmt)
    s = torch.ones(nO, dtype=torch.float32, device="cuda")
    s_ref = np.ones(nO, np.float32)
    Xq = torch.empty((M, K), dtype=torch.int8, device="cuda")
    a = torch.empty(M, dtype=torch.float32, device="cuda")
    XqO = torch.empty((M, nO), dtype=torch.int8, device="cuda")
    aws_n = q.qlin_quant_act_workspace(M, layer.w)
    aws = q.empty_workspace(aws_n)
    gws_n = q.qlin_gemm_workspace(M, layer.w)
    gws = q.empty_workspace(gws_n)
    Y = torch.empty((M, N), dtype=torch.float16, device="cuda")
    acc = torch.empty((M, N), dtype=torch.int32, device="cuda")
    rng = np.random.default_rng(20)
    assert wl.steps == 20
    for step in range(wl.steps):
        L = synth.layer(wl, si, M=M, step=step, with_weights=False)
        q.qlin_quant_act(torch.from_numpy(L["X"]).cuda(), M, layer.w, s, wl.gamma, True, Xq, a, XqO, aws, aws_n)
        q.qlin_gemm(layer.w, Xq, a, XqO, s, M, Y, acc, gws, gws_n)
        q.qlin_poll_device_status()
        torch.cuda.synchronize()
        a_gpu = a.cpu().numpy()
        rows = np.unique(np.concatenate([rng.choice(M, 16, replace=False),
                                         [int(np.argmax(a_gpu))]])).astype(np.int32)
        r = oracle.forward(bits(L["X"]), bits(W), pk, s_ref, wl.gamma, rows=rows)
        s_ref = r["s"]
        np.testing.assert_array_equal(s.cpu().numpy().view(np.uint32), s_ref.view(np.uint32), err_msg=f"s, step {step}")
        np.testing.assert_array_equal(Xq.cpu().numpy(), r["Xq"], err_msg=f"Xq, step {step}")
        np.testing.assert_array_equal(a_gpu.view(np.uint32), r["a"].view(np.uint32), err_msg=f"a, step {step}")
        np.testing.assert_array_equal(XqO.cpu().numpy(), r["XqO"], err_msg=f"XqO, step {step}")
        np.testing.assert_array_equal(acc.cpu().numpy()[rows].astype(np.int64), r["acc"], err_msg=f"acc, step {step}")
        y = Y.float().cpu().numpy().astype(np.float64)[rows]
        err = np.abs(y - r["y"]) / np.maximum(np.abs(r["y"]), 1.0)
        assert err.max() <= TOL, (step, err.max())
