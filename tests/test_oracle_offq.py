"""Pins of the oracle's OffQ path (the Hadamard offset, the per-group
asymmetric INT4 activations, the rotated weights and the per-group
product), each against a fact the method or the mathematics fixes."""
import numpy as np

from quantized_linear_layers_token_b200 import synth


def bits(a):
    return np.ascontiguousarray(a).view(np.uint16)


def test_transform_rows_orthogonal_first_row_ones(oracle):
    """The transform of the unit vectors are the rows of D H: they are
    orthogonal with squared norm 128, and the first is all ones (a value in
    channel 0 adds the same amount to every transformed channel)."""
    d = synth.offq_signs(3)
    E = np.eye(128, dtype=np.float16)
    R = oracle.offq_transform(bits(E), d)
    np.testing.assert_array_equal(R @ R.T, 128.0 * np.eye(128))
    np.testing.assert_array_equal(R[0], np.ones(128))
    assert set(np.unique(R)) == {-1.0, 1.0}


def test_outlier_becomes_offset(oracle):
    """A group whose first channel is an outlier: after the transform the
    outlier is a constant offset of the whole group, the group minimum
    carries it, and the INT4 grid step follows the small channels only --
    far finer than symmetric INT4 on the raw group."""
    rng = np.random.default_rng(4)
    x = rng.standard_normal((8, 256)).astype(np.float32)
    x[:, 0::128] = 900.0
    X = x.astype(np.float16)
    d = synth.offq_signs(1)
    Xq, sc, off = oracle.offq_quant_act(bits(X), d)
    y = oracle.offq_transform(bits(X), d)
    deq = Xq.astype(np.float64) * np.repeat(sc.astype(np.float64), 128, axis=1) + \
        np.repeat(off.astype(np.float64), 128, axis=1)
    assert np.abs(y - deq).max() <= 0.5 * sc.max() * (1 + 1e-4) + 1e-4
    assert (off > 800).all()  # the offset is the outlier
    # the grid step, brought back to the input's scale (the transform is
    # unnormalised: rows of norm sqrt(128)), is set by the small channels and
    # is far finer than a symmetric INT4 step over the raw group
    sym_step = np.abs(X.astype(np.float64)).reshape(8, 2, 128).max(axis=2) / 7.0
    assert (sc.astype(np.float64) / np.sqrt(128.0)).max() * 50 < sym_step.min()


def test_codes_are_nearest_grid_points(oracle):
    """Brute force: every code is the point of the group's 16-level grid
    lo + q sd, q in [0, 15], nearest to the transformed value (ties to even
    q); sd and lo from the group's range."""
    rng = np.random.default_rng(5)
    X = (rng.standard_normal((6, 384)) * rng.uniform(0.1, 30.0, (6, 1))).astype(np.float16)
    d = synth.offq_signs(2)
    Xq, sc, off = oracle.offq_quant_act(bits(X), d)
    y = oracle.offq_transform(bits(X), d)
    for m in range(6):
        for g in range(3):
            yg = y[m, g * 128:(g + 1) * 128]
            lo, hi = yg.min(), yg.max()
            sd = (hi - lo) / 15.0
            assert sc[m, g] == np.float32(sd) and off[m, g] == np.float32(lo)
            grid = lo + np.arange(16) * sd
            for j in range(128):
                dist = np.abs(yg[j] - grid)
                cand = np.flatnonzero(dist <= dist.min() * (1 + 1e-15))
                want = cand[0] if len(cand) == 1 else [c for c in cand if c % 2 == 0][0]
                assert Xq[m, g * 128 + j] == want, (m, g, j)


def test_constant_group_is_exact(oracle):
    """Only the outlier channel nonzero: the transformed group is constant,
    its step is 0 and the offset alone reproduces it."""
    X = np.zeros((2, 128), np.float16)
    X[:, 0] = 37.5
    Xq, sc, off = oracle.offq_quant_act(bits(X), synth.offq_signs(0))
    assert (sc == 0).all() and (Xq == 0).all() and (off == np.float32(37.5)).all()


def test_rotated_weights_preserve_the_product(oracle):
    """sum_g y_g W'_g = x W: pins the direction of the rotation (H D on the
    weight side) and the 1/128."""
    rng = np.random.default_rng(6)
    X = rng.standard_normal((5, 256)).astype(np.float16)
    W = (rng.standard_normal((256, 40)) * 0.05).astype(np.float16)
    d = synth.offq_signs(4)
    y = oracle.offq_transform(bits(X), d)
    pk = oracle.offq_pack_layer(bits(W), d)
    lhs = y @ pk["Wr"].astype(np.float64)
    rhs = X.astype(np.float64) @ W.astype(np.float64)
    assert np.abs(lhs - rhs).max() <= 1e-6 * np.abs(rhs).max()


def test_per_group_product_equals_dequantized_product(oracle):
    """The per-group integer product with the group's scale and offset
    equals the fp64 product of the dequantized activations and weights, and
    the layer's output stays close to x W."""
    rng = np.random.default_rng(7)
    X = synth.offq_activations(9, 384, seed=2)
    W = (rng.standard_normal((384, 48)) * 0.02).astype(np.float16)
    d = synth.offq_signs(5)
    Xq, sc, off = oracle.offq_quant_act(bits(X), d)
    pk = oracle.offq_pack_layer(bits(W), d)
    rows = np.arange(9, dtype=np.int32)
    y = oracle.offq_gemm_rows(Xq, sc, off, pk, rows)
    xd = Xq.astype(np.float64) * np.repeat(sc.astype(np.float64), 128, axis=1) + \
        np.repeat(off.astype(np.float64), 128, axis=1)
    wd = pk["q"].astype(np.float64) * pk["c"].astype(np.float64)[None, :]
    want = xd @ wd
    assert np.abs(y - want).max() <= 1e-12 * np.abs(want).max()
    ref = X.astype(np.float64) @ W.astype(np.float64)
    assert np.linalg.norm(y - ref) / np.linalg.norm(ref) < 0.15
