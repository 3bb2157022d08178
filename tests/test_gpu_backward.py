"""GPU parity of the input gradient (straight-through estimator, Quaff notes
损失函数 / 训练策略) against the oracle.

The kernel rounds Weff to fp16 and sums on the tensor cores in fp32, so the
bound per element is derived from that arithmetic:
  |dX - dX_oracle| <= sum_n |dY| (|Weff| + |W_deq|) (2^-10 + N 2^-22)   (Weff rounding, fp32 sums)
                      + 2^-11 |dX_oracle| + 2^-25                        (one fp16 rounding of dX;
                                                                          2^-25 below fp16's normal range)
                      + sum_n |dY| 2^-18 [c'_n below fp16's normal range]
A second check replays the kernel's fp16 rounding of Weff on the CPU and
holds the result to the much tighter bound of fp32 summation alone.
"""
import numpy as np
import pytest
import torch

from quantized_linear_layers_token_b200 import synth

pytestmark = pytest.mark.gpu
FMTS = [synth.W4_PERCHANNEL, synth.W4_G128, synth.W8_PERCHANNEL]


@pytest.fixture(scope="module")
def q():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from quantized_linear_layers_token_b200 import qlin
    qlin.lib()
    return qlin


def bits(a):
    return np.ascontiguousarray(a).view(np.uint16)


def w_eff(pk, W, s):
    """(Weff, W_deq) in fp64 [K][N] -- only to size the error bound."""
    Wd = pk["B"].astype(np.float64) * pk["cscale"].astype(np.float64)[None, :]
    We = Wd.copy()
    O = pk["O"]
    if len(O):
        sd = s.astype(np.float64)[:, None]
        We[O] = (Wd[O] + (sd - 1.0) * W[O].astype(np.float64)) / sd
    return We, Wd


def w_eff_fp16(pk, W, s):
    """Weff with the kernel's roundings: fp16(fp16(c') * B), outlier rows
    blended in fp32 from that value and rounded to fp16."""
    c16 = pk["cscale"].astype(np.float16)
    B16 = pk["B"].astype(np.float16)
    W16 = (B16 * c16[None, :]).astype(np.float16)
    O = pk["O"]
    if len(O):
        s32 = s.astype(np.float32)[:, None]
        bl = (W16[O].astype(np.float32) + (s32 - np.float32(1)) * W[O].astype(np.float32)) * (np.float32(1) / s32)
        W16[O] = bl.astype(np.float16)
    return W16.astype(np.float64)


def run(q, W, O, fmt, dY, s, workspace=False):
    """dX from the GPU; with workspace=True the tiles of an incomplete last
    wave are split along the reduction (fp32 partials through it), and the
    call is made twice to check that the workspace is left ready for reuse."""
    K, N = W.shape
    M = dY.shape[0]
    layer = q.PackedLayer.pack(torch.from_numpy(W).cuda(), O, fmt)
    dYd = torch.from_numpy(dY).cuda()
    sd = torch.from_numpy(s).cuda() if len(O) else None
    dX = torch.full((M, K), float("nan"), dtype=torch.float16, device="cuda")
    ws, nws = None, 0
    if workspace:
        nws = q.qlin_backward_dx_workspace(M, layer.w)
        ws = q.empty_workspace(nws) if nws else None
    q.qlin_backward_dx(layer.w, dYd, M, sd, dX, ws, nws)
    if workspace:
        first = dX.clone()
        dX.fill_(float("nan"))
        q.qlin_backward_dx(layer.w, dYd, M, sd, dX, ws, nws)
    q.qlin_poll_device_status()
    torch.cuda.synchronize()
    if workspace:
        assert torch.equal(first, dX), "second call with the same workspace differs"
        cnt = split_counters(ws, M, K, N) if ws is not None else None
        if cnt is not None:
            assert not cnt.any().item(), "split-tile counters not left zeroed"
    return dX.float().cpu().numpy().astype(np.float64)


def split_counters(ws, M, K, N):
    """The per-tile counters of the split plan (workspace layout: fp32
    partials of the split tiles, then one counter per split tile), or None
    when the call splits nothing."""
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    tiles = -(-K // 256) * -(-M // 256)
    tail = tiles % sms
    if tail == 0 or tiles >= 2 * sms:
        return None
    S = min(sms // tail, 8, -(-N // 64))
    if S < 2:
        return None
    cnt_off = -(-(tail * (S - 1) * 65536 * 4) // 256) * 256
    return ws[cnt_off:cnt_off + tail * 4]


def check(dX, dY, W, pk, s, oracle, rows=None):
    rows = np.arange(dY.shape[0]) if rows is None else rows
    dYr = dY[rows]
    ref = oracle.backward_dx(bits(dYr), bits(W), pk, s)
    got = dX[rows]
    assert np.all(np.isfinite(got))
    N = dY.shape[1]
    ady = np.abs(dYr.astype(np.float64))
    We, Wd = w_eff(pk, W, s)
    cs = pk["cscale"].astype(np.float64)
    subn = (ady * 2.0 ** -18 * (cs < 2.0 ** -14)[None, :]).sum(1, keepdims=True)
    bound = (ady @ (np.abs(We) + np.abs(Wd)).T * (2.0 ** -10 + N * 2.0 ** -22) + np.abs(ref) * 2.0 ** -11 + subn
             + 2.0 ** -25)
    err = np.abs(got - ref)
    assert np.all(err <= bound), ("oracle", float(err.max()), float((err / bound).max()))
    # the rounding model: only fp32 summation and the output rounding remain
    W16 = w_eff_fp16(pk, W, s)
    ref16 = dYr.astype(np.float64) @ W16.T
    tight = ady @ np.abs(W16).T * (N * 2.0 ** -22) + np.abs(ref16) * 2.0 ** -11 + 2.0 ** -25
    err16 = np.abs(got - ref16)
    assert np.all(err16 <= tight), ("fp16 model", float(err16.max()), float((err16 / tight).max()))


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("M,K,N,nO", [
    (200, 640, 208, 37),   # both 128-token halves (ragged), 3 input tiles (last half empty), ragged channel step
    (1, 256, 16, 0),       # one token, one 16-channel step, no outliers
    (129, 1152, 400, 64),  # one token past a 128-token half; odd number of code blocks
    (300, 384, 96, 11),    # two 256-token tiles, the second with its first half only
])
def test_backward_parity(q, oracle, fmt, M, K, N, nO):
    L = synth.layer("small", 0, M=1, K=K, N=N, n_outliers=nO)
    W, O = L["W"], L["O"]
    dY = synth.grad_output(0, 0, M, N)
    s = synth.outlier_scales(0, 0, nO)
    dX = run(q, W, O, fmt, dY, s)
    pk = oracle.pack_layer(bits(W), O, fmt)
    check(dX, dY, W, pk, s, oracle)


@pytest.mark.parametrize("fmt", FMTS)
def test_backward_dense_outliers(q, oracle, fmt):
    """Every input of the first tiles is an outlier (a full 256-entry table
    per tile), others at tile edges; scales below 1 included."""
    K, N, M = 1536, 144, 160
    O = np.unique(np.concatenate([np.arange(0, 512), [767, 768, 1023, 1024, 1279, 1535]])).astype(np.int32)
    L = synth.layer("small", 0, M=1, K=K, N=N, n_outliers=0)
    W = L["W"]
    s = synth.outlier_scales(0, 1, len(O), lo=0.5, hi=6.0)
    dY = synth.grad_output(0, 1, M, N)
    dX = run(q, W, O, fmt, dY, s)
    pk = oracle.pack_layer(bits(W), O, fmt)
    check(dX, dY, W, pk, s, oracle)


@pytest.mark.parametrize("wl_name,shape_idx", [
    ("llama7b_w4_decode", 0),         # q_proj 4096 -> 4096
    ("llama7b_w4g128_prefill", 4),    # gate_proj 4096 -> 11008
    ("phi3_w8_quaff", 3),             # down_proj 8192 -> 3072, 8% outliers
    ("llama7b_w4g128_prefill", 6),    # down_proj 11008 -> 4096
])
def test_backward_fullsize_sampled(q, oracle, wl_name, shape_idx):
    """Full-size layers at a fine-tuning token count; 6 sampled rows (one in
    each of the first and last token tiles) checked against the oracle."""
    wl = synth.WORKLOADS[wl_name]
    M = 2048
    L = synth.layer(wl, shape_idx, M=1)
    W, O = L["W"], L["O"]
    N = W.shape[1]
    dY = synth.grad_output(wl.index, shape_idx, M, N)
    s = synth.outlier_scales(wl.index, shape_idx, len(O))
    dX = run(q, W, O, wl.fmt, dY, s, workspace=True)
    pk = oracle.pack_layer(bits(W), O, wl.fmt)
    rows = np.array([0, 127, 700, 1301, 1920, M - 1])
    check(dX, dY, W, pk, s, oracle, rows=rows)


def test_backward_maximum_k(q, oracle):
    """K = 65536 with 4096 outliers, every format's largest supported layer
    shape along the reduction; 3 sampled rows."""
    K, N, M = 65536, 128, 130
    L = synth.layer("small", 0, M=1, K=K, N=N, n_outliers=4096)
    W, O = L["W"], L["O"]
    dY = synth.grad_output(0, 2, M, N)
    s = synth.outlier_scales(0, 2, len(O))
    for fmt in FMTS:
        dX = run(q, W, O, fmt, dY, s)
        pk = oracle.pack_layer(bits(W), O, fmt)
        check(dX, dY, W, pk, s, oracle, rows=np.array([0, 64, 129]))


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("M,K,N,nO", [
    (200, 640, 208, 37),    # 3 tiles: each split into ranges of the 4 channel steps
    (520, 1536, 1024, 41),  # 18 tiles, 8 ranges each (with a ragged token tile)
])
def test_backward_split_tiles(q, oracle, fmt, M, K, N, nO):
    """With a workspace, the tiles of an incomplete wave are split along the
    reduction; the last range adds the others' fp32 partials."""
    L = synth.layer("small", 0, M=1, K=K, N=N, n_outliers=nO)
    W, O = L["W"], L["O"]
    dY = synth.grad_output(0, 4, M, N)
    s = synth.outlier_scales(0, 4, nO)
    dX = run(q, W, O, fmt, dY, s, workspace=True)
    pk = oracle.pack_layer(bits(W), O, fmt)
    rows = np.unique(np.concatenate([np.arange(0, M, 37), [M - 1]])).astype(np.int64)
    check(dX, dY, W, pk, s, oracle, rows=rows)


def test_backward_zero_tokens_and_repeat(q):
    """M = 0 writes nothing; a second call on the same buffers gives the same
    bits (no state carried between calls)."""
    K, N, nO = 512, 256, 9
    L = synth.layer("small", 0, M=1, K=K, N=N, n_outliers=nO)
    layer = q.PackedLayer.pack(torch.from_numpy(L["W"]).cuda(), L["O"], synth.W8_PERCHANNEL)
    dY = torch.from_numpy(synth.grad_output(0, 3, 64, N)).cuda()
    s = torch.from_numpy(synth.outlier_scales(0, 3, nO)).cuda()
    dX = torch.full((64, K), 7.0, dtype=torch.float16, device="cuda")
    q.qlin_backward_dx(layer.w, dY, 0, s, dX)
    torch.cuda.synchronize()
    assert bool((dX == 7.0).all())
    q.qlin_backward_dx(layer.w, dY, 64, s, dX)
    a = dX.clone()
    q.qlin_backward_dx(layer.w, dY, 64, s, dX)
    q.qlin_poll_device_status()
    assert torch.equal(a, dX)
