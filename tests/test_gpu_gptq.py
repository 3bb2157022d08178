"""Hessian-compensated weight quantization on the GPU (qlin_gptq_quantize)
against the CPU oracle's layer form (itself pinned column for column to the
single-vector form, which the KKT, optimal-value and downdate pins hold).
Every fp64 step is the oracle's, in its order and without contraction, so
the compensated weights, the codes and the inverse Hessian are compared bit
for bit."""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def q():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from quantized_linear_layers_token_b200 import qlin
    qlin.lib()
    return qlin


def run_gpu(q, X, W, scale, qmax):
    ns, K = X.shape
    N = W.shape[1]
    Xd = torch.from_numpy(X).cuda()
    Wd = torch.from_numpy(np.ascontiguousarray(W)).cuda()
    sd = torch.from_numpy(scale).cuda()
    codes = torch.empty((K, N), dtype=torch.int8, device="cuda")
    Hinv = torch.empty((K, K), dtype=torch.float64, device="cuda")
    sing = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    n = q.qlin_gptq_workspace(K, N)
    ws = q.empty_workspace(n)
    q.qlin_gptq_quantize(Xd, ns, K, N, Wd, sd, qmax, codes, Hinv, sing, ws, n)
    q.qlin_poll_device_status()
    torch.cuda.synchronize()
    return Wd.cpu().numpy(), codes.cpu().numpy(), Hinv.cpu().numpy(), int(sing.item())


def calib(ns, K, N, seed, qmax):
    """Synthetic calibration activations with a few large channels (the
    outlier structure the layer's activations have) and N(0, 0.02) weights;
    per-channel grid steps max|W| / qmax."""
    rng = np.random.default_rng(seed)
    X = rng.standard_normal((ns, K))
    X[:, rng.choice(K, max(1, K // 100), replace=False)] *= 20.0
    W = rng.standard_normal((K, N)) * 0.02
    scale = np.abs(W).max(axis=0) / qmax
    return X, W, scale


@pytest.mark.parametrize("ns,K,N,qmax", [(40, 24, 7, 7), (512, 256, 96, 7), (300, 128, 130, 127),
                                         (2048, 1024, 256, 7)])
def test_gptq_matches_oracle_bitwise(q, oracle, ns, K, N, qmax):
    X, W, scale = calib(ns, K, N, K + N, qmax)
    Wg, cg, Hg, sing = run_gpu(q, X, W, scale, qmax)
    assert sing == 0
    Wo, co, Ho = oracle.gptq_quantize_layer(X, W, scale, qmax)
    np.testing.assert_array_equal(Hg.view(np.uint64), Ho.view(np.uint64))
    np.testing.assert_array_equal(cg, co)
    np.testing.assert_array_equal(Wg.view(np.uint64), Wo.view(np.uint64))


def test_gptq_singular_hessian_reported(q, oracle):
    X, W, scale = calib(64, 32, 8, 5, 7)
    X[:, 11] = 0.0  # a zero column: H has a zero row, the elimination meets a zero pivot
    *_, sing = run_gpu(q, X, W, scale, 7)
    assert sing == 1
    with pytest.raises(ValueError):
        oracle.gptq_quantize_layer(X, W, scale, 7)
