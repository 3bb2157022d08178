"""Host-side checks of the C ABI (no GPU needed): the library loads, exports
every entry point declared in include/qlin.h, and the host-only calls and
argument validation behave as documented (errors are returned before
anything is enqueued)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def q():
    from quantized_linear_layers_token_b200 import build, qlin
    build.build()
    return qlin


def declared_entry_points():
    with open(os.path.join(ROOT, "include", "qlin.h")) as f:
        text = f.read()
    return sorted(set(re.findall(r"QLIN_API\s+(?:const\s+char\s*\*|qlin_status)\s+(qlin_\w+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_entry_points()
    for must in ["qlin_pack_weights", "qlin_quant_act", "qlin_gemm", "qlin_forward"]:
        assert must in names


def test_library_exports_every_declared_symbol(q):
    L = ctypes.CDLL(q.LIB_PATH)
    for name in declared_entry_points():
        assert hasattr(L, name), name
    assert set(declared_entry_points()) <= set(q.EXPORTED) | {"qlin_status_string", "qlin_last_error"}


def test_status_strings(q):
    L = q.lib()
    for code, name in q.STATUS.items():
        assert L.qlin_status_string(code).decode() == name


def test_weights_bytes_and_bind(q):
    K, N, nO = 4096, 11008, 41
    for fmt in (0, 1, 2):
        n = q.qlin_weights_bytes(K, N, fmt, nO)
        codes = K * N if fmt == 2 else K * N // 2
        assert n >= codes + 4 * N + N * 48 * 2
        base = 1 << 20  # host-only: the descriptor is filled, memory untouched
        w = q.qlin_weights_bind(K, N, fmt, nO, base, n)
        assert (w.K, w.N, w.fmt, w.n_outlier, w.n_outlier_pad) == (K, N, fmt, nO, 48)
        assert w.group == (128 if fmt == 1 else 0)
        ptrs = [w.codes, w.chan_scale, w.outlier_idx, w.W_Ot, w.wmax_O]
        assert all(p % 256 == 0 and base <= p < base + n for p in ptrs)
        assert (w.group_scale is None) == (fmt != 1)


@pytest.mark.parametrize("K,N,fmt,nO,status", [
    (4100, 128, 0, 0, "QLIN_ERR_SHAPE"),   # K % 32
    (4096, 120, 0, 0, "QLIN_ERR_SHAPE"),   # N % 16
    (4064, 128, 1, 0, "QLIN_ERR_SHAPE"),   # g128 needs K % 128
    (512, 128, 7, 0, "QLIN_ERR_ARG"),      # unknown format
    (512, 128, 0, -1, "QLIN_ERR_ARG"),
    (512, 128, 0, 600, "QLIN_ERR_SHAPE"),  # more outliers than channels
    (65568, 128, 0, 0, "QLIN_ERR_SHAPE"),  # K above the supported 65536
    (8192, 128, 0, 4097, "QLIN_ERR_SHAPE"),  # more than 4096 outlier channels
    (0, 128, 0, 0, "QLIN_ERR_ARG"),
])
def test_shape_validation(q, K, N, fmt, nO, status):
    with pytest.raises(q.QlinError) as e:
        q.qlin_weights_bytes(K, N, fmt, nO)
    assert q.STATUS[e.value.status] == status


def test_pack_rejects_bad_outlier_sets(q):
    import numpy as np
    K, N, nO = 256, 128, 3
    n = q.qlin_weights_bytes(K, N, 0, nO)
    w = q.qlin_weights_bind(K, N, 0, nO, 1 << 20, n)
    fakeW = 1 << 24
    for O in ([5, 5, 9], [9, 5, 7], [1, 2, 256], [-1, 2, 3]):
        with pytest.raises(q.QlinError) as e:
            q.qlin_pack_weights(fakeW, np.array(O, np.int32), w, stream=0)
        assert q.STATUS[e.value.status] == "QLIN_ERR_ARG"
    with pytest.raises(q.QlinError) as e:
        q.qlin_pack_weights(fakeW + 8, np.array([1, 2, 3], np.int32), w, stream=0)
    assert q.STATUS[e.value.status] == "QLIN_ERR_ALIGN"


def test_workspace_and_alignment_errors(q):
    K, N, nO, M = 512, 128, 5, 16
    n = q.qlin_weights_bytes(K, N, 0, nO)
    w = q.qlin_weights_bind(K, N, 0, nO, 1 << 20, n)
    need = q.qlin_forward_workspace(M, w)
    assert need >= M * K + 4 * M + M * nO
    with pytest.raises(q.QlinError) as e:
        q.qlin_forward(1 << 24, M, w, 1 << 25, 0.9, True, 1 << 26, 1 << 27, need - 1, stream=0)
    assert q.STATUS[e.value.status] == "QLIN_ERR_WORKSPACE"
    with pytest.raises(q.QlinError) as e:
        q.qlin_gemm(w, (1 << 24) + 4, 1 << 25, 1 << 26, 1 << 27, M, 1 << 28, None, 1 << 29, 1 << 20, stream=0)
    assert q.STATUS[e.value.status] == "QLIN_ERR_ALIGN"
    with pytest.raises(q.QlinError) as e:
        q.qlin_quant_act(1 << 24, M, w, 1 << 25, 1.5, True, 1 << 26, 1 << 27, 1 << 28, 1 << 29, 4096, stream=0)
    assert q.STATUS[e.value.status] == "QLIN_ERR_ARG"  # gamma outside [0, 1]


def test_backward_argument_errors(q):
    K, N, nO = 512, 128, 5
    n = q.qlin_weights_bytes(K, N, 0, nO)
    w = q.qlin_weights_bind(K, N, 0, nO, 1 << 20, n)
    q.qlin_backward_dx(w, None, 0, None, None, stream=0)  # M = 0: nothing to do
    assert q.qlin_backward_dx_workspace(0, w) == 0
    # 4096 tokens x 512 inputs = 32 tiles < one wave: split, so a workspace is asked for
    assert q.qlin_backward_dx_workspace(4096, w) > 0
    for dY, M, s, status in [
        (1 << 24, -1, 1 << 25, "QLIN_ERR_ARG"),
        (None, 4, 1 << 25, "QLIN_ERR_ARG"),
        (1 << 24, 4, None, "QLIN_ERR_ARG"),  # s is needed when the layer has outliers
        ((1 << 24) + 2, 4, 1 << 25, "QLIN_ERR_ALIGN"),
        (1 << 24, 65535 * 128 + 1, 1 << 25, "QLIN_ERR_SHAPE"),
    ]:
        with pytest.raises(q.QlinError) as e:
            q.qlin_backward_dx(w, dY, M, s, 1 << 26, stream=0)
        assert q.STATUS[e.value.status] == status
    with pytest.raises(q.QlinError) as e:  # a workspace off the 256-byte grid
        q.qlin_backward_dx(w, 1 << 24, 4, 1 << 25, 1 << 26, (1 << 27) + 16, 1 << 20, stream=0)
    assert q.STATUS[e.value.status] == "QLIN_ERR_ALIGN"


def test_offq_argument_errors(q):
    """OffQ shapes, signs and sizes are checked on the host before anything
    is enqueued."""
    import numpy as np
    from quantized_linear_layers_token_b200 import synth
    d = synth.offq_signs(0)
    assert q.qlin_offq_codes_bytes(256, 160) == 2 * 2 * 8192
    assert q.qlin_offq_gemm_workspace(7, 256, 160) == 2 * 2 * 16384
    assert q.qlin_offq_forward_workspace(7, 256, 160) > q.qlin_offq_gemm_workspace(7, 256, 160)
    q.qlin_offq_quant_act(None, 0, 256, d, None, None, None, stream=0)  # M = 0: nothing to do
    for K, N, status in [(200, 128, "QLIN_ERR_SHAPE"), (256, 120, "QLIN_ERR_SHAPE"), (0, 128, "QLIN_ERR_ARG"),
                         (65536 + 128, 128, "QLIN_ERR_SHAPE")]:
        with pytest.raises(q.QlinError) as e:
            q.qlin_offq_codes_bytes(K, N)
        assert q.STATUS[e.value.status] == status
    bad = d.copy()
    bad[0] = -1  # row 0 of D H must be all ones
    half = d.copy()
    half[5] = 0
    for signs in (bad, half):
        with pytest.raises(q.QlinError) as e:
            q.qlin_offq_quant_act(1 << 24, 4, 256, signs, 1 << 25, 1 << 26, 1 << 27, stream=0)
        assert q.STATUS[e.value.status] == "QLIN_ERR_ARG"
    with pytest.raises(q.QlinError) as e:
        q.qlin_offq_quant_act((1 << 24) + 8, 4, 256, d, 1 << 25, 1 << 26, 1 << 27, stream=0)
    assert q.STATUS[e.value.status] == "QLIN_ERR_ALIGN"
    with pytest.raises(q.QlinError) as e:
        q.qlin_offq_gemm(1 << 24, 1 << 25, 1 << 26, 4, 256, 160, 1 << 27, 1 << 28, 1 << 29, 1 << 30, 1 << 31,
                         16, stream=0)
    assert q.STATUS[e.value.status] == "QLIN_ERR_WORKSPACE"
    with pytest.raises(ValueError):
        q.qlin_offq_quant_act(1 << 24, 4, 256, np.ones(64, np.int8), 1 << 25, 1 << 26, 1 << 27, stream=0)


def test_binding_declares_every_entry_point(q):
    """Every entry point of the header has an argument list in the ctypes
    binding (so no call goes out with default int conversions)."""
    L = q.lib()
    for name in declared_entry_points():
        if name in ("qlin_status_string", "qlin_last_error"):
            continue
        assert getattr(L, name).argtypes is not None, name


def test_synthetic_inputs_are_reproducible():
    """Both sides of every parity test draw the same arrays from the seeded
    generator: repeated draws are identical, different shapes independent."""
    import numpy as np
    from quantized_linear_layers_token_b200 import synth
    a = synth.layer("llama7b_w4_decode", 0, M=4)
    b = synth.layer("llama7b_w4_decode", 0, M=4)
    for k in ("X", "W", "O"):
        assert np.array_equal(a[k], b[k])
    c = synth.layer("llama7b_w4_decode", 1, M=4)
    assert not np.array_equal(a["W"], c["W"])
    assert np.array_equal(synth.grad_output(1, 0, 8, 64), synth.grad_output(1, 0, 8, 64))
    assert np.array_equal(synth.outlier_scales(1, 0, 5), synth.outlier_scales(1, 0, 5))


def header_knobs():
    with open(os.path.join(ROOT, "include", "qlin.h")) as f:
        text = f.read()
    return {m.group(1): int(m.group(2)) for m in re.finditer(r"\b(QLIN_KNOB_\w+)\s*=\s*(\d+)", text)}


def test_knob_ids_match_the_header(q):
    knobs = header_knobs()
    assert knobs, "no knob enum in the header"
    for name, value in knobs.items():
        assert getattr(q, name) == value, name


# documented defaults (include/qlin.h, test and measurement hooks)
KNOB_DEFAULTS = {"PDL": 1, "CLUSTER": 1, "CLUSTER_SIZE": 0, "MAX_CTAS": 0, "MAX_TOKEN_TILE": 256,
                 "WIDEN_MIN_M": 512, "FUSED_MOMENTUM_MAX_M": 64, "WAIT_NS": 2000000000, "PAIR_MMA": 2,
                 "CONVERT_MAX_M": 0, "PAIR_SPLIT": 0}


def test_knob_defaults_and_validation(q):
    for name, value in KNOB_DEFAULTS.items():
        assert q.qlin_debug_get(getattr(q, "QLIN_KNOB_" + name)) == value, name
    bad = [("PDL", 2), ("CLUSTER", -1), ("CLUSTER_SIZE", 3), ("MAX_TOKEN_TILE", 32), ("PAIR_MMA", 3),
           ("PAIR_SPLIT", 2), ("MAX_CTAS", -1), ("WIDEN_MIN_M", -5)]
    for name, value in bad:
        k = getattr(q, "QLIN_KNOB_" + name)
        with pytest.raises(q.QlinError):
            q.qlin_debug_set(k, value)
        assert q.qlin_debug_get(k) == KNOB_DEFAULTS[name], name  # a refused value leaves the knob as it was
    for k in (-1, max(header_knobs().values()) + 1):
        with pytest.raises(q.QlinError):
            q.qlin_debug_set(k, 0)
        with pytest.raises(q.QlinError):
            q.qlin_debug_get(k)


def test_knobs_context_restores(q):
    with q.knobs(pair_split=1, widen_min_m=129, pair_mma=1):
        assert q.qlin_debug_get(q.QLIN_KNOB_PAIR_SPLIT) == 1
        assert q.qlin_debug_get(q.QLIN_KNOB_WIDEN_MIN_M) == 129
        with q.knobs(pair_split=0):
            assert q.qlin_debug_get(q.QLIN_KNOB_PAIR_SPLIT) == 0
        assert q.qlin_debug_get(q.QLIN_KNOB_PAIR_SPLIT) == 1
    for name in ("PAIR_SPLIT", "WIDEN_MIN_M", "PAIR_MMA"):
        assert q.qlin_debug_get(getattr(q, "QLIN_KNOB_" + name)) == KNOB_DEFAULTS[name]
