"""QQQ adaptive smoothing threshold search on the GPU (qlin_smooth_search)
against the CPU oracle: every candidate's loss within 1e-3 relative (the
GPU sums the unquantized reference in fp32, the oracle in fp64; the
quantized product is exact on both sides), the same best candidate unless
the oracle's two best losses are closer than that, and the returned
smoothing vector of the best candidate exact."""
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


def case(M, K, N, seed):
    rng = np.random.default_rng(seed)
    X = rng.standard_normal((M, K)).astype(np.float32)
    X[:, rng.choice(K, max(2, K // 50), replace=False)] *= rng.uniform(20, 80)
    W = (rng.standard_normal((K, N)) * 0.02).astype(np.float32)
    return X.astype(np.float16), W.astype(np.float16)


@pytest.mark.parametrize("M,K,N,G", [(64, 512, 256, 8), (128, 1024, 384, 6), (37, 256, 128, 5)])
def test_smooth_search_matches_oracle(q, oracle, M, K, N, G):
    X, W = case(M, K, N, M + K)
    loss = torch.zeros(G, dtype=torch.float64, device="cuda")
    best = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    s_best = torch.zeros(K, dtype=torch.float32, device="cuda")
    n = q.qlin_smooth_search_workspace(M, K, N, G)
    ws = q.empty_workspace(n)
    for _ in range(2):  # the workspace is reused as the first call left it
        q.qlin_smooth_search(torch.from_numpy(X).cuda(), M, K, torch.from_numpy(W).cuda(), N, G, loss, best,
                             s_best, ws, n)
    q.qlin_poll_device_status()
    torch.cuda.synchronize()
    lo, bo = oracle.smooth_search(X.view(np.uint16), W.view(np.uint16), G)
    lg = loss.cpu().numpy()
    np.testing.assert_allclose(lg, lo, rtol=1e-3)
    bg = int(best.item())
    order = np.argsort(lo)
    if abs(lo[order[1]] - lo[order[0]]) > 2e-3 * lo[order[0]]:
        assert bg == bo
    # the smoothing vector of the GPU's choice: sqrt(cmax / wmax) on T, 1 elsewhere
    x32, w32 = X.astype(np.float32), W.astype(np.float32)
    cmax = np.abs(x32).max(axis=0)
    wmax = np.abs(w32).max(axis=1)
    sigma = np.float32(np.float32(cmax.max() * np.float32(bg)) / np.float32(G))
    inT = cmax > sigma
    want = np.where(inT & (cmax > 0) & (wmax > 0), np.sqrt(cmax / np.where(wmax > 0, wmax, 1)), 1).astype(np.float32)
    np.testing.assert_array_equal(s_best.cpu().numpy().view(np.uint32), want.view(np.uint32))
