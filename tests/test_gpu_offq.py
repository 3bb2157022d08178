"""OffQ on the GPU against the CPU oracle.

Bit-exact: the activation codes, group scales and offsets (the transform is
exact in fp64 on both sides and every rounding decision is taken in fp64),
the rotated fp32 weights, the packed INT4 codes, the channel scales and the
per-group column sums.  The output Y: the GPU sums the groups' promoted
products in fp32 (two fused multiply-adds per group) and rounds to fp16, the
oracle sums in fp64; the bound per element is

    |Y - y| <= 2^-11 |y| + 2^-24 (2 G + 4) (c_n / 16) T[m][n] + 2^-24,

with T = sum_k (sd q[m][k] + |lo|) |16 q_w[k][n]| (the terms' magnitudes;
2^-11 is the fp16 half-ulp, the second term the fp32 sum, the last the fp16
subnormal spacing)."""
import numpy as np
import pytest
import torch

from quantized_linear_layers_token_b200 import synth

from layouts import tile_w4

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def q():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from quantized_linear_layers_token_b200 import qlin
    qlin.lib()
    return qlin


def bits(a):
    return np.ascontiguousarray(a).view(np.uint16)


def pz(a):
    """Floats with -0.0 folded into +0.0, as bit patterns."""
    return (np.asarray(a, np.float32) + np.float32(0.0)).view(np.uint32)


def gpu_pack(q, W, d):
    K, N = W.shape
    codes = torch.zeros(q.qlin_offq_codes_bytes(K, N), dtype=torch.uint8, device="cuda")
    cs = torch.zeros(N, dtype=torch.float32, device="cuda")
    colsum = torch.zeros((K // 128, N), dtype=torch.float32, device="cuda")
    Wr = torch.zeros((K, N), dtype=torch.float32, device="cuda")
    q.qlin_offq_pack(torch.from_numpy(bits(W)).cuda(), K, N, d, codes, cs, colsum, Wr)
    return codes, cs, colsum, Wr


def gpu_quant(q, X, d):
    M, K = X.shape
    Xq = torch.full((M, K), -1, dtype=torch.int8, device="cuda")
    sc = torch.full((M, K // 128), -1.0, dtype=torch.float32, device="cuda")
    off = torch.full((M, K // 128), -1.0, dtype=torch.float32, device="cuda")
    q.qlin_offq_quant_act(torch.from_numpy(bits(X)).cuda(), M, K, d, Xq, sc, off)
    return Xq, sc, off


def bound(oracle_q, sc, off, layer, rows):
    """Per-element tolerance of the module docstring for the given rows."""
    B = layer["B"].astype(np.float64)  # [K][N], 16 q_w
    K = B.shape[0]
    G = K // 128
    A = oracle_q[rows].astype(np.float64) * np.repeat(sc[rows].astype(np.float64), 128, axis=1) + \
        np.repeat(np.abs(off[rows].astype(np.float64)), 128, axis=1)
    T = A @ np.abs(B)
    c = layer["c"].astype(np.float64) / 16.0
    return 2.0 ** -24 * (2 * G + 4) * c[None, :] * T + 2.0 ** -24


def check_y(Y, y_ref, tol):
    Y = Y.astype(np.float64)
    err = np.abs(Y - y_ref)
    lim = 2.0 ** -11 * np.abs(y_ref) + tol
    bad = err > lim
    assert not bad.any(), f"{bad.sum()} elements out of bound; worst excess {(err - lim).max()}"
    # the layer-level bar of the W4A8 path holds too
    assert (err / np.maximum(np.abs(y_ref), 1.0)).max() <= 2e-3


def with_edge_rows(X):
    """Ragged extras: an all-zero token, a token whose groups are constant
    after the transform (only each group's first channel nonzero), and one
    tiny-magnitude token (fp16 subnormals)."""
    X = X.copy()
    if X.shape[0] >= 3:
        X[0] = 0
        X[1] = 0
        X[1, 0::128] = np.float16(37.5)
        X[2] = (X[2].astype(np.float32) * np.float32(2.0 ** -20)).astype(np.float16)
    return X


QUANT_SHAPES = [(1, 128), (3, 256), (37, 512), (300, 1024), (129, 384)]


@pytest.mark.parametrize("M,K", QUANT_SHAPES)
def test_quant_act_bit_exact(q, oracle, M, K):
    d = synth.offq_signs(M)
    X = with_edge_rows(synth.offq_activations(M, K, seed=K))
    Xq, sc, off = gpu_quant(q, X, d)
    torch.cuda.synchronize()
    oq, osc, ooff = oracle.offq_quant_act(bits(X), d)
    np.testing.assert_array_equal(Xq.cpu().numpy(), oq)
    np.testing.assert_array_equal(pz(sc.cpu().numpy()), pz(osc))
    np.testing.assert_array_equal(pz(off.cpu().numpy()), pz(ooff))
    if M >= 3:
        assert (osc[1] == 0).all() and (oq[1] == 0).all()  # the constant groups


PACK_SHAPES = [(128, 16), (256, 160), (512, 384), (1024, 272)]


@pytest.mark.parametrize("K,N", PACK_SHAPES)
def test_pack_bit_exact(q, oracle, K, N):
    d = synth.offq_signs(K + N)
    W = synth.offq_weights(K, N, seed=N)
    codes, cs, colsum, Wr = gpu_pack(q, W, d)
    torch.cuda.synchronize()
    L = oracle.offq_pack_layer(bits(W), d)
    np.testing.assert_array_equal(Wr.cpu().numpy().view(np.uint32), L["Wr"].view(np.uint32))
    np.testing.assert_array_equal(codes.cpu().numpy(), tile_w4(L["packed"], N, K))
    np.testing.assert_array_equal(cs.cpu().numpy().view(np.uint32), L["c"].view(np.uint32))
    want = L["B"].astype(np.int64).reshape(K // 128, 128, N).sum(axis=1)
    np.testing.assert_array_equal(colsum.cpu().numpy(), want.astype(np.float32))


GEMM_SHAPES = [(1, 128, 128), (37, 256, 160), (129, 512, 272), (300, 1024, 384), (256, 384, 128)]


@pytest.mark.parametrize("M,K,N", GEMM_SHAPES)
def test_gemm_matches_oracle(q, oracle, M, K, N):
    """Full parity of every output at sizes spanning several tiles and ragged
    token and channel tails, through both entry points (the GEMM alone on
    quantized activations, and the whole forward), each called twice on the
    same workspace."""
    d = synth.offq_signs(7)
    X = with_edge_rows(synth.offq_activations(M, K, seed=M))
    W = synth.offq_weights(K, N, seed=K)
    codes, cs, colsum, _ = gpu_pack(q, W, d)
    Xq, sc, off = gpu_quant(q, X, d)
    Y1 = torch.full((M, N), 0x7E00, dtype=torch.int16, device="cuda")
    Y2 = torch.full((M, N), 0x7E00, dtype=torch.int16, device="cuda")
    n1 = q.qlin_offq_gemm_workspace(M, K, N)
    ws1 = q.empty_workspace(n1)
    n2 = q.qlin_offq_forward_workspace(M, K, N)
    ws2 = q.empty_workspace(n2)
    for _ in range(2):
        q.qlin_offq_gemm(Xq, sc, off, M, K, N, codes, cs, colsum, Y1, ws1, n1)
        q.qlin_offq_forward(torch.from_numpy(bits(X)).cuda(), M, K, N, d, codes, cs, colsum, Y2, ws2, n2)
    q.qlin_poll_device_status()
    torch.cuda.synchronize()
    oq, osc, ooff = oracle.offq_quant_act(bits(X), d)
    L = oracle.offq_pack_layer(bits(W), d)
    rows = np.arange(M, dtype=np.int32)
    y_ref = oracle.offq_gemm_rows(oq, osc, ooff, L, rows)
    tol = bound(oq, osc, ooff, L, rows)
    Yg1 = Y1.cpu().numpy().view(np.float16)
    Yg2 = Y2.cpu().numpy().view(np.float16)
    check_y(Yg1, y_ref, tol)
    np.testing.assert_array_equal(Yg1.view(np.uint16), Yg2.view(np.uint16))


FULL = [
    ("llama3_8b q_proj", 4096, 4096, 4096),
    ("llama3_8b k_proj", 4096, 4096, 1024),
]


@pytest.mark.parametrize("name,M,K,N", FULL)
def test_fullsize_sampled(q, oracle, name, M, K, N):
    """The bench's launch configuration (prefill, 4096 tokens): every code
    and scale of the sampled tokens bit-exact, and their outputs within the
    bound; sampled rows are seeded plus the first and last token."""
    d = synth.offq_signs(11)
    X = synth.offq_activations(M, K, seed=3)
    W = synth.offq_weights(K, N, seed=4)
    codes, cs, colsum, _ = gpu_pack(q, W, d)
    Xq, sc, off = gpu_quant(q, X, d)
    Y = torch.full((M, N), 0x7E00, dtype=torch.int16, device="cuda")
    n = q.qlin_offq_gemm_workspace(M, K, N)
    ws = q.empty_workspace(n)
    q.qlin_offq_gemm(Xq, sc, off, M, K, N, codes, cs, colsum, Y, ws, n)
    q.qlin_poll_device_status()
    torch.cuda.synchronize()
    rng = np.random.default_rng(M + N)
    rows = np.unique(np.concatenate([[0, M - 1], rng.choice(M, 14, replace=False)])).astype(np.int32)
    oq, osc, ooff = oracle.offq_quant_act(bits(X[rows]), d)
    np.testing.assert_array_equal(Xq.cpu().numpy()[rows], oq)
    np.testing.assert_array_equal(pz(sc.cpu().numpy()[rows]), pz(osc))
    np.testing.assert_array_equal(pz(off.cpu().numpy()[rows]), pz(ooff))
    L = oracle.offq_pack_layer(bits(W), d)
    np.testing.assert_array_equal(cs.cpu().numpy().view(np.uint32), L["c"].view(np.uint32))
    local = np.arange(len(rows), dtype=np.int32)
    y_ref = oracle.offq_gemm_rows(oq, osc, ooff, L, local)
    tol = bound(oq, osc, ooff, L, local)
    check_y(Y.cpu().numpy().view(np.float16)[rows], y_ref, tol)
