"""The GEMM's work split is chosen per call (global stream-K, or cluster
split-K with 2, 4 or 8 CTAs per tile), INT4 weights are widened ahead of
the GEMM for large token counts, many-token tiles run on CTA pairs, and
kernels are chained with programmatic dependent launch.  The library's test knobs (qlin_debug_set)
force each variant, so every one of them is checked against the oracle
here: the exact INT32 accumulators of the split-K test and the ragged-shape
sweep, with the knob set for the duration of the test only."""
import pytest
import torch

from quantized_linear_layers_token_b200 import synth
from test_gpu_fullsize import run_full_forward as _run_full_forward
from test_gpu_fullsize import test_split_k_accumulators_exact as _split_k_case
from test_gpu_parity import test_shapes as _shape_case, SHAPES
from test_gpu_parity import case as _case, run_gpu as _run_gpu
import numpy as np

pytestmark = pytest.mark.gpu

MODES = [
    {"cluster": 0},            # global stream-K for every split tile
    {"cluster_size": 2},
    {"cluster_size": 4},
    {"cluster_size": 8},
    {"pdl": 0},                # plain stream-ordered launches
    {"widen_min_m": 129},      # INT4 weights widened once, INT8 kernel, from 129 tokens
    {"widen_min_m": 0},        # INT4 converters in the GEMM for every token count
    {"pair_mma": 2, "widen_min_m": 129},  # CTA-pair GEMM for every 256-token tile with INT8 operands
    {"pair_mma": 2, "widen_min_m": 129, "pair_split": 1},  # ... with the stream-K tail
    {"pair_mma": 1, "widen_min_m": 1024},  # CTA pairs only from a full wave of pair tiles
    {"pair_mma": 0},           # one CTA per tile everywhere
    {"convert_max_m": 1 << 20, "widen_min_m": 129},  # INT4 on CTA pairs, converted inside the GEMM
]


@pytest.fixture(scope="module")
def q():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from quantized_linear_layers_token_b200 import qlin
    qlin.lib()
    return qlin


@pytest.mark.parametrize("mode", MODES, ids=lambda e: ",".join(f"{k}={v}" for k, v in e.items()))
def test_forced_split_mode(q, oracle, mode):
    with q.knobs(**mode):
        for fmt in (0, 1, 2):
            for M in (1, 16, 48):
                _split_k_case(q, oracle, fmt, M)
        for args in SHAPES:
            _shape_case(q, oracle, *args)


@pytest.mark.parametrize("wl_name,shape_idx,ms", [
    ("llama70b_w4g128", 2, [1024]),       # up_proj 8192 -> 28672
    ("llama7b_w4g128_prefill", 6, [512]),  # down_proj 11008 -> 4096
    ("llama7b_w4_decode", 4, [512]),       # per-channel INT4, gate_proj 4096 -> 11008 (86 channel tiles)
])
def test_pair_convert_full_size(q, oracle, wl_name, shape_idx, ms):
    """INT4 layers on CTA pairs with the codes converted inside the GEMM, at
    bench sizes: codes, scales and accumulators bit-exact on sampled rows."""
    with q.knobs(convert_max_m=1 << 20):
        _run_full_forward(q, oracle, synth.WORKLOADS[wl_name], shape_idx, ms)


@pytest.mark.parametrize("fmt,M,K,N,nO", [
    (2, 700, 512, 384, 17),     # 6 pair tiles on every pair: each tile split into many short ranges
    (1, 1000, 4096, 1536, 40),  # g128 widened: 24 tiles, ranges of a few K-blocks
    (0, 2304, 1024, 4096, 0),   # per-channel widened, no outliers: 144 tiles (a wave and a partial one)
    (2, 4096, 2048, 2560, 70),  # 160 tiles: the last full wave and the remainder split
])
def test_pair_stream_k_matches_whole_tiles(q, oracle, fmt, M, K, N, nO):
    """The stream-K tail of CTA-pair launches sums exact INT32 partials (and
    takes each tile's compensation from the one range that holds it): the
    accumulators and Y are bit-identical to the same launch with whole tiles,
    and the accumulators equal the oracle's."""
    L = _case(fmt, M, K, N, nO, seed_shape=0)
    rng = np.random.default_rng(M + K + N)
    s0 = rng.uniform(1.0, 4.0, nO).astype(np.float32)
    with q.knobs(widen_min_m=129, pair_split=0):
        whole = _run_gpu(q, L, s0, 0.9, with_forward=False)
        with q.knobs(pair_split=1):
            split = _run_gpu(q, L, s0, 0.9, with_forward=False)
    np.testing.assert_array_equal(split["acc"].cpu().numpy(), whole["acc"].cpu().numpy())
    np.testing.assert_array_equal(split["Y"].cpu().numpy().view(np.uint16), whole["Y"].cpu().numpy().view(np.uint16))
    # accumulators of sampled rows against the oracle's integer product on
    # the same codes (the codes themselves are checked in the parity tests)
    rows = np.unique(np.r_[0, M - 1, rng.integers(0, M, 6)]).astype(np.int32)
    pk = oracle.pack_layer(np.ascontiguousarray(L["W"]).view(np.uint16), L["O"], fmt)
    want, ovf = oracle.int_gemm_rows(split["Xq"].cpu().numpy(), pk["B"], rows)
    assert ovf == 0
    np.testing.assert_array_equal(split["acc"].cpu().numpy()[rows].astype(np.int64), want)
