"""Pins of the oracle's input gradient under the straight-through estimator
(Quaff notes, 损失函数 / 训练策略: standard STE backpropagation; 解耦 WAQ
公式 for the layer the gradient passes through)."""
import numpy as np
import pytest

from quantized_linear_layers_token_b200 import synth

FMTS = [synth.W4_PERCHANNEL, synth.W4_G128, synth.W8_PERCHANNEL]


def bits(a):
    return np.ascontiguousarray(a).view(np.uint16)


def _layer(fmt, M, K, N, nO, seed):
    L = synth.layer("small", 0, M=M, K=K, N=N, n_outliers=nO)
    rng = np.random.default_rng(seed)
    dY = rng.standard_normal((M, N)).astype(np.float16)
    s = rng.uniform(1.0, 5.0, nO).astype(np.float32)
    return L, dY, s


def _forward_map(X, W, pk, s):
    """The decoupled layer the estimator differentiates, written forward:
    X_hat = X / s (outlier columns), Y = X_hat W_deq + X_hat[:, O] (s_O - 1) W_O."""
    K = X.shape[1]
    O = pk["O"]
    sd = np.ones(K)
    sd[O] = s
    Xh = X / sd
    W_deq = pk["B"].astype(np.float64) * pk["cscale"].astype(np.float64)[None, :]
    W_O = W.astype(np.float64)[O, :]
    return Xh @ W_deq + (Xh[:, O] * (s.astype(np.float64) - 1.0)) @ W_O


@pytest.mark.parametrize("fmt", FMTS)
def test_adjoint_identity(oracle, fmt):
    # <dY, F(X)> = <dX, X> for the linear map F: dX is exactly its transpose
    M, K, N, nO = 5, 256, 96, 9
    L, dY, s = _layer(fmt, M, K, N, nO, 11 + fmt)
    pk = oracle.pack_layer(bits(L["W"]), L["O"], fmt)
    dX = oracle.backward_dx(bits(dY), bits(L["W"]), pk, s)
    rng = np.random.default_rng(5)
    for _ in range(3):
        X = rng.standard_normal((M, K))
        lhs = np.sum(dY.astype(np.float64) * _forward_map(X, L["W"], pk, s))
        rhs = np.sum(dX * X)
        # fp64 rounding of two differently ordered sums of ~M*N*K terms
        scale = np.abs(dY.astype(np.float64)).sum() * np.abs(X).sum() * np.abs(pk["cscale"]).max() * 256
        assert abs(lhs - rhs) <= 1e-13 * scale


@pytest.mark.parametrize("fmt", FMTS)
def test_unit_scale_is_dequantized_matmul(oracle, fmt):
    # s = 1: the compensation vanishes and dX = dY W_deq^T (a library matmul)
    M, K, N, nO = 4, 384, 160, 7
    L, dY, _ = _layer(fmt, M, K, N, nO, 3)
    pk = oracle.pack_layer(bits(L["W"]), L["O"], fmt)
    dX = oracle.backward_dx(bits(dY), bits(L["W"]), pk, np.ones(nO, np.float32))
    W_deq = pk["B"].astype(np.float64) * pk["cscale"].astype(np.float64)[None, :]
    ref = dY.astype(np.float64) @ W_deq.T
    np.testing.assert_allclose(dX, ref, rtol=1e-12, atol=1e-12)


def test_close_to_unquantized_gradient(oracle):
    # W8, s = 1: |W_deq - W| <= c_n / 2 elementwise, so
    # |dX - dY W^T| <= sum_n |dY| c_n / 2 (the textbook gradient of X W)
    M, K, N, nO = 3, 512, 128, 5
    L, dY, _ = _layer(synth.W8_PERCHANNEL, M, K, N, nO, 8)
    pk = oracle.pack_layer(bits(L["W"]), L["O"], synth.W8_PERCHANNEL)
    dX = oracle.backward_dx(bits(dY), bits(L["W"]), pk, np.ones(nO, np.float32))
    ref = dY.astype(np.float64) @ L["W"].astype(np.float64).T
    bound = (np.abs(dY.astype(np.float64)) @ (pk["c"].astype(np.float64) / 2))[:, None]
    assert np.all(np.abs(dX - ref) <= bound * (1 + 1e-9) + 1e-12)


def test_no_outliers_and_empty(oracle):
    L, dY, _ = _layer(synth.W4_PERCHANNEL, 2, 128, 64, 0, 1)
    pk = oracle.pack_layer(bits(L["W"]), L["O"], synth.W4_PERCHANNEL)
    dX = oracle.backward_dx(bits(dY), bits(L["W"]), pk, np.zeros(0, np.float32))
    W_deq = pk["B"].astype(np.float64) * pk["cscale"].astype(np.float64)[None, :]
    np.testing.assert_allclose(dX, dY.astype(np.float64) @ W_deq.T, rtol=1e-12, atol=1e-12)
    dX0 = oracle.backward_dx(np.zeros((0, 64), np.uint16), bits(L["W"]), pk, np.zeros(0, np.float32))
    assert dX0.shape == (0, 128)
