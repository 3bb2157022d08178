"""Pins for the CPU oracle: each test checks the oracle against something
other than itself -- a library routine, brute-force enumeration, a closed
form or an algebraic identity of the pages -- so that a dropped term, a wrong
sign or index or a transposed operand in the oracle fails here.

Sources: the Quaff notes page ("解耦 WAQ 公式", "目标动量缩放") and the QQQ
review page ("Hessian补偿", "W4A8 GEMM内核": per-channel GEMM, per-group GEMM,
FusedDequantQuant, FastFP16toINT8).
"""
import numpy as np
import pytest

from quantized_linear_layers_token_b200 import synth


def f16_bits(x):
    with np.errstate(over="ignore"):  # values past the fp16 range round to infinity, as intended
        return np.ascontiguousarray(np.asarray(x, np.float16)).view(np.uint16)


# ---------------------------------------------------------------------------
# binary16 conversions against numpy's IEEE binary16
# ---------------------------------------------------------------------------

def test_half_decode_all_patterns(oracle):
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    got = np.array([oracle.half_to_double(int(b)) for b in bits])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])
    # signed zeros keep their sign
    assert np.array_equal(np.signbit(got[~nan]), np.signbit(ref[~nan]))


def test_half_encode_matches_numpy(oracle):
    rng = np.random.default_rng(7)
    xs = np.concatenate([
        rng.standard_normal(20000) * 10.0 ** rng.integers(-9, 6, 20000),
        rng.uniform(-70000, 70000, 2000),
        # exact ties between neighbouring halves, normal and subnormal
        (np.arange(1, 2000, dtype=np.float64) + 0.5) * 2.0 ** -24,
        (np.arange(1024, 3072, dtype=np.float64) + 0.5) * 2.0 ** -10,
        np.array([65504.0, 65519.99, 65520.0, 1e6, -65520.0, 2.0 ** -25, 2.0 ** -26, 0.0, -0.0]),
    ])
    ref = f16_bits(xs)  # numpy rounds double -> half to nearest, ties to even
    got = np.array([oracle.double_to_half(float(x)) for x in xs], np.uint16)
    assert np.array_equal(got, ref)
    xf = xs.astype(np.float32)
    got32 = np.array([oracle.float_to_half(x) for x in xf], np.uint16)
    assert np.array_equal(got32, f16_bits(xf))


def test_rne_enumeration(oracle):
    # ties go to the even neighbour; everything else to the nearest integer
    for k in range(-300, 300):
        for frac, want in [(0.5, k if k % 2 == 0 else k + 1), (0.25, k), (0.75, k + 1),
                           (0.49999999, k), (0.50000001, k + 1)]:
            assert oracle.rne(k + frac) == want, (k, frac)


# ---------------------------------------------------------------------------
# helpers for the brute-force pins
# ---------------------------------------------------------------------------

def nearest_code_ok(t: np.ndarray, q: np.ndarray, qmax: int, tie_tol: float = 2e-6):
    """q must be the integer in [-qmax, qmax] nearest to t (t exact in fp64),
    found by enumerating every candidate; exact ties go to the even one.
    When t is within tie_tol (relative) of a half-integer the fp32 rounding of
    the scaled value may fall either side, and both neighbours are accepted."""
    cands = np.arange(-qmax, qmax + 1, dtype=np.float64)
    err = np.abs(t.reshape(-1, 1) - cands.reshape(1, -1))
    best = err.min(axis=1)
    q = q.reshape(-1).astype(np.float64)
    qerr = np.abs(t.reshape(-1) - q)
    near_tie = np.abs(np.abs(t.reshape(-1) - np.floor(t.reshape(-1))) - 0.5) <= tie_tol * np.maximum(1, np.abs(t.reshape(-1)))
    ok_exact = qerr == best
    # among exact ties prefer even
    tie_mask = (np.sum(err == best.reshape(-1, 1), axis=1) == 2) & ok_exact
    ok_even = ~tie_mask | (q % 2 == 0)
    ok_near = near_tie & (qerr <= best + 1.0) & (np.abs(q) <= qmax)
    return (ok_exact & ok_even) | ok_near


def xhat_f32(X16, O, s):
    x = X16.astype(np.float32)
    if len(O):
        x[:, O] = x[:, O] / s.astype(np.float32)[None, :]
    return x


# ---------------------------------------------------------------------------
# P1: brute force on 4x8x8 inputs, >= 10^4 seeded draws
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("fmt", [synth.W4_PERCHANNEL, synth.W8_PERCHANNEL])
def test_bruteforce_4x8x8(oracle, fmt):
    rng = np.random.default_rng(1234 + fmt)
    M, K, N = 4, 8, 8
    draws = 5000
    for d in range(draws):
        nO = int(rng.integers(0, 4))
        O = np.sort(rng.choice(K, nO, replace=False)).astype(np.int32)
        X = rng.standard_normal((M, K)).astype(np.float32)
        X[:, O] *= rng.uniform(20, 100, nO).astype(np.float32)
        if d % 97 == 0:
            X[rng.integers(0, M)] = 0.0  # an all-zero token
        X16 = X.astype(np.float16)
        W16 = (rng.standard_normal((K, N)) * 0.02).astype(np.float16)
        if d % 89 == 0:
            W16[:, rng.integers(0, N)] = 0  # an all-zero output channel
        Wb = f16_bits(W16)
        pk = oracle.pack_layer(Wb, O, fmt)
        s0 = rng.uniform(1.0, 3.0, nO).astype(np.float32)
        r = oracle.forward(f16_bits(X16), Wb, pk, s0, float(rng.uniform(0, 1)))
        s1 = r["s"]
        assert np.all(s1 >= 1.0)
        # (a) activation codes: nearest integer to x_hat * 127 / amax
        xh = xhat_f32(X16, O, s1).astype(np.float64)
        amax = np.abs(xh).max(axis=1)
        assert np.array_equal(r["a"], (amax.astype(np.float32) / np.float32(127)))
        t = np.where(amax[:, None] > 0, xh * 127.0 / np.where(amax > 0, amax, 1)[:, None], 0.0)
        assert nearest_code_ok(t, r["Xq"], 127).all()
        assert np.array_equal(r["XqO"], r["Xq"][:, O])
        # weight codes: nearest integer to w * qmax / wmax
        qmax = 7 if fmt == synth.W4_PERCHANNEL else 127
        w = W16.astype(np.float64)
        wmax = np.abs(w).max(axis=0)
        tw = np.where(wmax[None, :] > 0, w * qmax / np.where(wmax > 0, wmax, 1)[None, :], 0.0)
        assert nearest_code_ok(tw, pk["q"], qmax).all()
        # (b) the integer path equals "dequantize, then fp64 matmul"
        xd = r["Xq"].astype(np.float64) * r["a"].astype(np.float64)[:, None]
        if fmt == synth.W4_PERCHANNEL:
            wd = pk["q"].astype(np.float64) * pk["c"].astype(np.float64)[None, :]
        else:
            wd = pk["q"].astype(np.float64) * pk["c"].astype(np.float64)[None, :]
        y_alt = xd @ wd
        if nO:
            y_alt += (xd[:, O] * (s1.astype(np.float64) - 1.0)[None, :]) @ w[O, :]
        assert np.allclose(r["y"], y_alt, rtol=1e-12, atol=1e-12 * max(1.0, np.abs(y_alt).max()))


def test_bruteforce_g128_codes(oracle):
    """Per-group path on small blocks: every q4 is the nearest code on the
    group grid, every q8 is the nearest integer to q4 * r exactly, r is g/c
    rounded once to fp16, c is 7 * max g / 127."""
    rng = np.random.default_rng(99)
    for d in range(40):
        K, N = 256, 8
        W16 = (rng.standard_normal((K, N)) * 0.02).astype(np.float16)
        spikes = rng.choice(K * N, 5, replace=False)
        W16.reshape(-1)[spikes] *= np.float16(20)
        if d == 3:
            W16[0:128, 2] = 0  # an all-zero group
        if d == 4:
            W16[:, 5] = 0  # an all-zero channel
        q4, q8, gh, rh, c, bad = oracle.quant_weight_group(f16_bits(W16), 128)
        assert bad == 0
        ghf = gh.view(np.float16).astype(np.float64)
        rhf = rh.view(np.float16).astype(np.float64)
        w = W16.astype(np.float64)
        for j in range(K // 128):
            blk = w[j * 128:(j + 1) * 128]
            gmax = np.abs(blk).max(axis=0)
            # g_h is fp16(fp32(gmax / 7)): within half an fp16 ulp of gmax/7 (plus fp32 rounding)
            np.testing.assert_allclose(ghf[j], gmax / 7.0, rtol=2 ** -11 + 2 ** -23, atol=2 ** -25)
            t = np.where(ghf[j][None, :] > 0, blk / np.where(ghf[j] > 0, ghf[j], 1)[None, :], 0.0)
            assert nearest_code_ok(t, q4[j * 128:(j + 1) * 128], 7).all()
            # q8: nearest integer to the exact product q4 * r, ties to even
            prod = q4[j * 128:(j + 1) * 128].astype(np.float64) * rhf[j][None, :]
            assert nearest_code_ok(prod, q8[j * 128:(j + 1) * 128], 127, tie_tol=0).all()
        cmax = ghf.max(axis=0)
        np.testing.assert_allclose(c, 7.0 * cmax / 127.0, rtol=2 ** -22)
        ratio = np.where(c[None, :] > 0, ghf / np.where(c > 0, c, 1)[None, :].astype(np.float64), 0.0)
        np.testing.assert_allclose(rhf, ratio, rtol=2 ** -11 + 2 ** -22)
        assert np.abs(q8.astype(np.int32)).max() <= 127


# ---------------------------------------------------------------------------
# P2: (16q) * (s/16) == q * s exactly, and acc(16q) == 16 * acc(q)
# ---------------------------------------------------------------------------

def test_shift4_scale_exact(oracle):
    rng = np.random.default_rng(5)
    s = (rng.standard_normal(1_000_000) * 10.0 ** rng.integers(-6, 6, 1_000_000)).astype(np.float32)
    s = s[np.abs(s) > 1e-30]
    for q in range(-8, 8):
        lhs = np.float32(16 * q) * (s / np.float32(16))
        rhs = np.float32(q) * s
        assert np.array_equal(lhs.view(np.uint32), rhs.view(np.uint32)), q
    Xq = rng.integers(-127, 128, (5, 64)).astype(np.int8)
    q = rng.integers(-7, 8, (64, 9)).astype(np.int8)
    acc1, _ = oracle.int_gemm(Xq, q)
    acc16, _ = oracle.int_gemm(Xq, (q.astype(np.int16) * 16).astype(np.int8))
    assert np.array_equal(acc16, 16 * acc1)
    assert np.array_equal(acc1, Xq.astype(np.int64) @ q.astype(np.int64))


def test_nibble_layout_shift_property(oracle):
    """The packed layout makes (w << 4) & 0xF0F0F0F0 the int8 lanes 16*q[k0..k0+3]
    and w & 0xF0F0F0F0 the lanes 16*q[k0+4..k0+7] (the per-channel <<4 unpack)."""
    rng = np.random.default_rng(11)
    K, N = 64, 5
    q = rng.integers(-8, 8, (K, N)).astype(np.int8)
    packed = oracle.pack_nibbles(q)
    assert packed.shape == (N, K // 2)
    words = packed.view(np.uint32)  # little-endian words, [N][K/8]
    for n in range(N):
        for wi in range(K // 8):
            w = int(words[n, wi])
            lo = ((w << 4) & 0xF0F0F0F0).to_bytes(4, "little")
            hi = (w & 0xF0F0F0F0).to_bytes(4, "little")
            lo_i8 = np.frombuffer(lo, np.int8).astype(np.int32)
            hi_i8 = np.frombuffer(hi, np.int8).astype(np.int32)
            k0 = wi * 8
            assert np.array_equal(lo_i8, 16 * q[k0:k0 + 4, n].astype(np.int32))
            assert np.array_equal(hi_i8, 16 * q[k0 + 4:k0 + 8, n].astype(np.int32))


# ---------------------------------------------------------------------------
# P3 / P4: the decoupled WAQ identity and the sparsity of (s - 1)
# ---------------------------------------------------------------------------

def test_decoupling_identity_fp64():
    rng = np.random.default_rng(3)
    M, K, N = 6, 40, 12
    X = rng.standard_normal((M, K)) * 50
    W = rng.standard_normal((K, N)) * 0.02
    O = np.sort(rng.choice(K, 5, replace=False))
    s = np.ones(K)
    s[O] = rng.uniform(1, 30, len(O))
    Xh = X / s[None, :]
    lhs = Xh @ (s[:, None] * W)
    rhs = Xh @ W + (Xh[:, O] * (s[O] - 1)[None, :]) @ W[O, :]
    np.testing.assert_allclose(lhs, rhs, rtol=1e-12, atol=1e-12 * np.abs(lhs).max())
    np.testing.assert_allclose(Xh @ (s[:, None] * W), X @ W, rtol=1e-12, atol=1e-12 * np.abs(lhs).max())


def test_oracle_epilogue_matches_identity(oracle):
    """With unit scales and integer weights exactly representable in fp16 the
    oracle's y equals Xq . diag(s') . B with s' = s on O and 1 elsewhere."""
    rng = np.random.default_rng(4)
    M, K, N = 5, 48, 7
    Xq = rng.integers(-127, 128, (M, K)).astype(np.int8)
    B = rng.integers(-127, 128, (K, N)).astype(np.int8)
    O = np.sort(rng.choice(K, 6, replace=False)).astype(np.int32)
    s = rng.uniform(1, 9, len(O)).astype(np.float32)
    acc, _ = oracle.int_gemm(Xq, B)
    y = oracle.dequant(acc, np.ones(M, np.float32), np.ones(N, np.float32),
                       np.ascontiguousarray(Xq[:, O]), s, f16_bits(B.astype(np.float16)), O)
    sfull = np.ones(K)
    sfull[O] = s.astype(np.float64)
    ref = Xq.astype(np.float64) @ (sfull[:, None] * B.astype(np.float64))
    np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-9)


def test_compensation_dense_equals_sparse(oracle):
    """(s - 1) vanishes off O: the compensation over every channel (s = 1 off
    O) equals the compensation over O only, bit for bit."""
    rng = np.random.default_rng(8)
    M, K, N = 4, 32, 6
    Xq = rng.integers(-127, 128, (M, K)).astype(np.int8)
    W16 = (rng.standard_normal((K, N)) * 0.02).astype(np.float16)
    O = np.sort(rng.choice(K, 4, replace=False)).astype(np.int32)
    s = rng.uniform(1, 9, len(O)).astype(np.float32)
    acc = rng.integers(-10 ** 6, 10 ** 6, (M, N)).astype(np.int64)
    a = rng.uniform(0.01, 0.1, M).astype(np.float32)
    c = rng.uniform(0.001, 0.01, N).astype(np.float32)
    y_sparse = oracle.dequant(acc, a, c, np.ascontiguousarray(Xq[:, O]), s, f16_bits(W16), O)
    Oall = np.arange(K, dtype=np.int32)
    sall = np.ones(K, np.float32)
    sall[O] = s
    y_dense = oracle.dequant(acc, a, c, Xq, sall, f16_bits(W16), Oall)
    assert np.array_equal(y_sparse.view(np.uint64), y_dense.view(np.uint64))


# ---------------------------------------------------------------------------
# P5: FastFP16toINT8, exhaustively over every fp16 value in [-128, 127]
# ---------------------------------------------------------------------------

def test_fast_fp16_to_int8_exhaustive(oracle):
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    vals = bits.view(np.float16).astype(np.float64)
    sel = np.isfinite(vals) & (vals >= -128) & (vals <= 127)
    vb = bits[sel]
    vv = vals[sel]
    assert len(vb) == 45042
    want = np.rint(vv).astype(np.int64)  # numpy rint: nearest, ties to even
    single = np.array([oracle.fast_fp16_to_int8(int(b), True) for b in vb])
    assert np.array_equal(single[:, 0], want)
    assert np.all(single[:, 1] == 0x64)
    two = np.array([oracle.fast_fp16_to_int8(int(b), False) for b in vb])
    mism = int(np.sum(two[:, 0] != want))
    # The literal two-add reading rounds twice; report how often it differs.
    print(f"two-add FastFP16toINT8 mismatches vs RNE: {mism} of {len(vb)}")
    assert np.all(two[:, 1] == 0x64)


# ---------------------------------------------------------------------------
# P6: GPTQ / QQQ Hessian compensation against its closed form (4x4)
# ---------------------------------------------------------------------------

def test_gptq_closed_form_4x4(oracle):
    rng = np.random.default_rng(21)
    for trial in range(50):
        X = rng.standard_normal((16, 4))
        H = oracle.gptq_hessian(X)
        np.testing.assert_allclose(H, 2 * X.T @ X, rtol=1e-13, atol=1e-12)
        Hinv = np.linalg.inv(H)
        w = rng.standard_normal(4)
        i = int(rng.integers(0, 4))
        q_i = float(np.round(w[i] * 4) / 4)
        delta = oracle.gptq_delta(w, Hinv, i, q_i)
        # constraint: the i-th weight lands on its quantized value
        assert abs((w[i] + delta[i]) - q_i) < 1e-12
        # KKT of  min d^T H d  s.t.  e_i^T d = q_i - w_i   (direct 5x5 solve)
        A = np.zeros((5, 5))
        A[:4, :4] = 2 * H
        A[:4, 4] = A[4, :4] = np.eye(4)[i]
        rhs = np.zeros(5)
        rhs[4] = q_i - w[i]
        kkt = np.linalg.solve(A, rhs)[:4]
        np.testing.assert_allclose(delta, kkt, rtol=1e-10, atol=1e-12)
        # optimal value: d^T H d == (w_i - Q(w_i))^2 / [H^-1]_ii
        np.testing.assert_allclose(delta @ H @ delta, (w[i] - q_i) ** 2 / Hinv[i, i], rtol=1e-10,
                                   atol=1e-14)
        # sequential downdate == inverse of H with row/column i removed
        Hd = oracle.gptq_downdate(Hinv, i)
        keep = [j for j in range(4) if j != i]
        np.testing.assert_allclose(Hd[np.ix_(keep, keep)], np.linalg.inv(H[np.ix_(keep, keep)]),
                                   rtol=1e-9, atol=1e-12)
        assert np.allclose(Hd[i, :], 0, atol=1e-12) and np.allclose(Hd[:, i], 0, atol=1e-12)


def test_gptq_sequential_equals_greedy_least_squares(oracle):
    """Full sequential pass against its definition by direct minimisation:
    at step i, with columns < i fixed on the grid, the free columns take the
    least-squares minimiser of ||X (w' - w)||^2 (numpy lstsq), and column i
    is rounded from there.  The oracle's delta + downdate recursion must land
    on the same grid points."""
    rng = np.random.default_rng(22)
    for t in range(40):
        d = 4
        X = rng.standard_normal((64, d)) @ rng.standard_normal((d, d))
        w = rng.standard_normal(d)
        scale = 0.25
        wq, Hinv, deltas = oracle.gptq_quantize(X, w, scale, 7)
        fixed = []
        for i in range(d):
            free = list(range(i, d))
            # minimise ||X[:, free] v - (X w - X[:, fixed] q_fixed)||
            target = X @ w - (X[:, :i] @ np.array(fixed) if i else 0.0)
            v, *_ = np.linalg.lstsq(X[:, free], target, rcond=None)
            fixed.append(float(np.clip(np.rint(v[0] / scale), -7, 7) * scale))
        np.testing.assert_allclose(wq, np.array(fixed), atol=1e-9)


# ---------------------------------------------------------------------------
# P7: momentum recurrence closed form
# ---------------------------------------------------------------------------

def test_momentum_closed_form(oracle):
    K, N = 16, 8
    O = np.array([2, 5, 11], np.int32)
    W = np.zeros((K, N), np.float16)
    W[O, 0] = np.float16(0.25)  # wmax = 0.25 for each outlier row
    W[3, 1] = np.float16(1.0)
    wmax = oracle.outlier_wmax(f16_bits(W), O)
    assert np.array_equal(wmax, np.full(3, 0.25, np.float32))
    X = np.zeros((3, K), np.float16)
    X[1, 2] = 4.0     # cmax/wmax = 16 -> beta = 4
    X[0, 5] = -1.0    # cmax/wmax = 4  -> beta = 2
    X[2, 11] = 0.125  # cmax/wmax = 0.5 -> beta = 1 (floor at 1)
    beta = np.array([4.0, 2.0, 1.0])
    Xb = f16_bits(X)
    for gamma in [0.0, 0.5, 0.9, 0.99]:
        s = np.ones(3, np.float32)
        for t in range(1, 21):
            s = oracle.momentum_update(Xb, O, wmax, gamma, s)
            closed = beta + gamma ** t * (1.0 - beta)
            np.testing.assert_allclose(s, closed, rtol=2e-6)
            assert np.all(s >= 1.0)
        if gamma == 0.0:
            assert np.array_equal(s, beta.astype(np.float32))
    s0 = np.array([1.5, 3.0, 7.0], np.float32)
    assert np.array_equal(oracle.momentum_update(Xb, O, wmax, 1.0, s0), s0)


# ---------------------------------------------------------------------------
# P8 / P9: rounding error bound and the |q8| <= 127 obligation on real shapes
# ---------------------------------------------------------------------------

def test_rounding_error_bound_small_workload(oracle):
    L = synth.layer("small", 0)
    Xb, Wb, O = f16_bits(L["X"]), f16_bits(L["W"]), L["O"]
    pk = oracle.pack_layer(Wb, O, synth.W4_PERCHANNEL)
    r = oracle.forward(Xb, Wb, pk, np.ones(len(O), np.float32), L["gamma"])
    xh = xhat_f32(L["X"], O, r["s"]).astype(np.float64)
    a = r["a"].astype(np.float64)
    err = np.abs(xh - r["Xq"].astype(np.float64) * a[:, None])
    assert np.all(err <= a[:, None] / 2 * (1 + 1e-6))
    w = L["W"].astype(np.float64)
    c = pk["c"].astype(np.float64)
    errw = np.abs(w - pk["q"].astype(np.float64) * c[None, :])
    assert np.all(errw <= c[None, :] / 2 * (1 + 1e-6))


@pytest.mark.parametrize("wl,shape", [("llama7b_w4g128_prefill", 0), ("llama7b_w4g128_prefill", 4),
                                      ("llama70b_w4g128", 1)])
def test_g128_requant_codes_in_range(oracle, wl, shape):
    L = synth.layer(wl, shape, M=1)
    q4, q8, gh, rh, c, bad = oracle.quant_weight_group(f16_bits(L["W"]), 128)
    assert bad == 0
    assert np.abs(q8.astype(np.int32)).max() <= 127
    assert np.abs(q4.astype(np.int32)).max() <= 7


def test_quant_act_zero_row_and_empty_O(oracle):
    X = np.zeros((3, 16), np.float16)
    X[1] = np.linspace(-3, 3, 16)
    Xq, a, XqO = oracle.quant_act(f16_bits(X), np.zeros(0, np.int32), np.zeros(0, np.float32))
    assert a[0] == 0 and a[2] == 0 and not Xq[0].any() and not Xq[2].any()
    assert a[1] == np.float32(3.0) / np.float32(127)
    assert Xq[1, 0] == -127 and Xq[1, -1] == 127
    assert XqO.shape == (3, 0)


def test_oracle_regression_fixture(oracle):
    """The oracle's output on the small workload is unchanged since the
    fixture was written (tests/golden/make_golden.py calls only the oracle)."""
    import json
    import os
    import sys
    here = os.path.join(os.path.dirname(__file__), "golden")
    sys.path.insert(0, here)
    import make_golden
    with open(os.path.join(here, "small_oracle.json")) as f:
        stored = json.load(f)["cases"]
    now = make_golden.compute()
    assert now == stored


def test_int_gemm_row_forms_agree_with_numpy(oracle):
    """The row GEMM over the transposed operand (the form the full-size
    parity checks use) equals numpy's exact int64 matmul, and so the plain
    form, including sums that reach the int32 range edge."""
    rng = np.random.default_rng(77)
    for K, N in [(64, 48), (1024, 96), (8192, 16)]:
        Xq = rng.integers(-127, 128, (5, K)).astype(np.int8)
        B = rng.integers(-127, 128, (K, N)).astype(np.int8)
        Xq[0] = 127
        B[:, 0] = 127  # the largest positive sum
        rows = np.array([4, 0, 2], np.int32)
        want = Xq[rows].astype(np.int64) @ B.astype(np.int64)
        acc_kn, _ = oracle.int_gemm_rows(Xq, B, rows)
        acc_nk, _ = oracle.int_gemm_rows_nk(Xq, np.ascontiguousarray(B.T), rows)
        np.testing.assert_array_equal(acc_kn, want)
        np.testing.assert_array_equal(acc_nk, want)


def test_gptq_layer_equals_row_by_row(oracle):
    """The layer form of the Hessian compensation (one shared inverse and
    downdate sequence) gives, column for column, exactly what the pinned
    single-vector form gives, and codes * scale are the grid values."""
    rng = np.random.default_rng(9)
    ns, d, N, qmax = 40, 24, 7, 7
    X = rng.standard_normal((ns, d))
    W = rng.standard_normal((d, N)) * 0.1
    scale = np.abs(W).max(axis=0) / qmax
    Wq, codes, Hinv = oracle.gptq_quantize_layer(X, W, scale, qmax)
    for n in range(N):
        w_row, Hinv_row, _ = oracle.gptq_quantize(X, W[:, n], float(scale[n]), qmax)
        np.testing.assert_array_equal(Wq[:, n], w_row)
        np.testing.assert_array_equal(Hinv, Hinv_row)
    np.testing.assert_array_equal(codes.astype(np.float64) * scale[None, :], Wq)
    assert np.abs(codes).max() <= qmax
    # the compensation lowers the layer's output error against plain rounding
    plain = np.clip(np.rint(W / scale), -qmax, qmax) * scale
    err_gptq = np.linalg.norm(X @ (Wq - W))
    err_plain = np.linalg.norm(X @ (plain - W))
    assert err_gptq < err_plain


def _smooth_case(M, K, N, seed):
    rng = np.random.default_rng(seed)
    X = rng.standard_normal((M, K)).astype(np.float32)
    X[:, rng.choice(K, max(2, K // 50), replace=False)] *= rng.uniform(20, 80)
    W = (rng.standard_normal((K, N)) * 0.02).astype(np.float32)
    return X.astype(np.float16), W.astype(np.float16)


def test_smooth_search_composes_pinned_quantizers(oracle):
    """Each candidate's loss equals the same steps assembled from the pinned
    quantizers (per-token INT8, per-channel INT4), numpy's exact integer
    matmul and an fp64 reference on the smoothed channel set; the search
    returns the first least loss."""
    X, W = _smooth_case(12, 64, 24, 3)
    G = 6
    loss, best = oracle.smooth_search(X.view(np.uint16), W.view(np.uint16), G)
    assert best == int(np.argmin(loss)) and (loss >= 0).all()
    x32, w32 = X.astype(np.float32), W.astype(np.float32)
    cmax = np.abs(x32).max(axis=0)
    wmax = np.abs(w32).max(axis=1)
    xall = np.float32(cmax.max())
    for j in range(G):
        sigma = np.float32(np.float32(xall * np.float32(j)) / np.float32(G))
        inT = cmax > sigma
        s = np.where(inT & (cmax > 0) & (wmax > 0), np.sqrt(cmax / np.where(wmax > 0, wmax, 1)), np.float32(1))
        s = s.astype(np.float32)
        Xh = np.where(inT[None, :], x32 / s[None, :], 0).astype(np.float16)
        Wh = np.where(inT[:, None], w32 * s[:, None], 0).astype(np.float16)
        xq, a, _ = oracle.quant_act(Xh.view(np.uint16), np.zeros(0, np.int32), np.zeros(0, np.float32))
        q, c = oracle.quant_weight_per_channel(Wh.view(np.uint16), 7)
        acc = xq.astype(np.int64) @ (16 * q.astype(np.int64))
        y = acc.astype(np.float64) * a.astype(np.float64)[:, None] * (c.astype(np.float64) / 16.0)[None, :]
        ref = X.astype(np.float64)[:, inT] @ W.astype(np.float64)[inT, :]
        want = float(((y - ref) ** 2).sum())
        assert abs(loss[j] - want) <= 1e-12 * want, (j, loss[j], want)


def test_smooth_search_channel_permutation_invariant(oracle):
    """Relabelling the input channels (columns of X with the rows of W) does
    not change any candidate's loss: a mixed-up index (a column maximum taken
    over the wrong axis, a factor applied to the wrong channel) would."""
    X, W = _smooth_case(10, 96, 16, 8)
    perm = np.random.default_rng(1).permutation(96)
    l1, b1 = oracle.smooth_search(X.view(np.uint16), W.view(np.uint16), 5)
    l2, b2 = oracle.smooth_search(np.ascontiguousarray(X[:, perm]).view(np.uint16),
                                  np.ascontiguousarray(W[perm, :]).view(np.uint16), 5)
    np.testing.assert_allclose(l1, l2, rtol=1e-12)
    assert b1 == b2
