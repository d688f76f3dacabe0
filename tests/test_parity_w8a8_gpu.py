"""GPU parity of the W8A8 path (the INT8 path that the Keras guide "INT4
quantization in Keras", section "How it works", says its INT4 steps extend)
against the CPU oracle on the same seeded inputs.

Bars as for the INT4 layer: weight codes, weight scales and the INT32
accumulator bit-exact; float32 output within 1e-6 relative (plus |bias|);
bfloat16 output within 1 ulp of the oracle's bf16 rounding.
"""
import numpy as np
import pytest
import torch

import oracle
from tests.test_parity_gpu import assert_bf16_within_ulp, assert_f32_close, dev, host
from w4a8_quantized_gemm_channel_b200 import synth

pytestmark = pytest.mark.gpu

PATHS = ["generic", "decode", "tc"]


@pytest.fixture(scope="module")
def nat():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from w4a8_quantized_gemm_channel_b200 import native
    native.get_device_status(clear=True)
    yield native
    assert native.get_device_status() == 0, "a kernel recorded an internal fault"


def _case(m, k, n, seed, outliers=4):
    w = synth.linear_weights(k, n, 0.02, seed)
    x, _ = synth.linear_activations(m, k, seed, outlier_count=min(outliers, k), outlier_factor=20.0)
    b = synth.bias_vector(n, seed)
    return x, w, b


@pytest.mark.parametrize("k,n", [(1, 1), (10, 32), (33, 7), (130, 45), (1152, 256), (4096, 130)])
def test_w8_quantize_bit_exact(nat, k, n):
    w = synth.linear_weights(k, n, 0.02, seed=2000 + k + n)
    if n > 3:
        w[:, 3] = 0.0  # an all-zero column: scale 1, codes 0
    q8, sw = oracle.w8_quantize(w)
    wqd, swd = nat.w8_quantize(dev(w))
    assert np.array_equal(host(wqd), q8)
    assert np.array_equal(host(swd).view(np.uint32), sw.view(np.uint32))


@pytest.mark.parametrize("k,n", [(1, 32), (257, 40), (4097, 96), (12288, 32), (12289, 32)])
def test_w8_quantize_panel_path_bit_exact(nat, k, n):
    """Shapes around the single-pass (cluster panel) form's limits, as for the
    INT4 weights: a partial panel, a last slice past K, K = 12288 and the first
    K handed to the two-pass form."""
    w = synth.linear_weights(k, n, 0.02, seed=2050 + k + n)
    w[:, 3] = 0.0
    w[k // 2, 5] = 0.5
    q8, sw = oracle.w8_quantize(w)
    wqd, swd = nat.w8_quantize(dev(w))
    assert np.array_equal(host(wqd), q8)
    assert np.array_equal(host(swd).view(np.uint32), sw.view(np.uint32))


def test_w8_quantize_wide_stride_writes_zero_pad(nat):
    """Rows wider than round_up(K, 16): every byte from K on is written 0."""
    k, n = 37, 20
    w = synth.linear_weights(k, n, 0.02, seed=2010)
    wq = torch.full((n, 96), 77, dtype=torch.int8, device="cuda")
    nat.w8_quantize(dev(w), wq=wq)
    q8, _ = oracle.w8_quantize(w, ldw8=96)
    assert np.array_equal(host(wq), q8)
    # aligned layout (single-pass form) with a row stride past the cluster's rows
    k, n = 300, 32
    w = synth.linear_weights(k, n, 0.02, seed=2011)
    wq = torch.full((n, 1024), 77, dtype=torch.int8, device="cuda")
    nat.w8_quantize(dev(w), wq=wq)
    q8, _ = oracle.w8_quantize(w, ldw8=1024)
    assert np.array_equal(host(wq), q8)


@pytest.mark.parametrize("path", PATHS)
@pytest.mark.parametrize("m,k,n", [(1, 64, 16), (3, 33, 17), (8, 256, 40), (16, 4096, 64),
                                   (17, 300, 33), (40, 1000, 130), (300, 520, 300),
                                   (256, 4096, 1024)])
def test_w8a8_s32_bit_exact(nat, path, m, k, n):
    x, w, _ = _case(m, k, n, seed=2100 + m + k + n)
    q8, sw = oracle.w8_quantize(w)
    acc = nat.w8a8_linear(dev(x), dev(q8), dev(sw), out="s32", path=path)
    assert nat.last_path() == path
    assert np.array_equal(host(acc), oracle.linear8(x, q8, sw, k, out="s32"))


@pytest.mark.parametrize("path", PATHS)
@pytest.mark.parametrize("relu", [False, True])
def test_w8a8_f32_bf16_bias_relu(nat, path, relu):
    m, k, n = 37, 700, 150
    x, w, b = _case(m, k, n, seed=2200)
    x[5] = 0.0  # a zero row: scale 1, codes 0, output = bias (then ReLU)
    q8, sw = oracle.w8_quantize(w)
    xd, qd, sd, bd = dev(x), dev(q8), dev(sw), dev(b)
    y = nat.w8a8_linear(xd, qd, sd, bias=bd, relu=relu, path=path)
    assert_f32_close(host(y), oracle.linear8(x, q8, sw, k, bias=b, relu=relu), b)
    yb = nat.w8a8_linear(xd, qd, sd, bias=bd, relu=relu, out="bf16", path=path)
    assert_bf16_within_ulp(host(yb.view(torch.int16)), oracle.linear8(x, q8, sw, k, bias=b, relu=relu, out="bf16"))


@pytest.mark.parametrize("path", PATHS)
def test_w8a8_q_ignores_activation_pad_bytes(nat, path):
    """INT8 input with a row stride past K: the pad bytes multiply zero weight
    pad and must not change the result; the same bits as w8a8_linear."""
    m, k, n = 20, 100, 48
    x, w, b = _case(m, k, n, seed=2300)
    q8, sw = oracle.w8_quantize(w)
    xq, sx = oracle.a8_quantize_rows(x, ldq=128)
    xq[:, k:] = -99
    y = nat.w8a8_linear_q(dev(xq), dev(sx), k, dev(q8), dev(sw), bias=dev(b), path=path)
    ref = oracle.linear8_q(xq[:, :k], sx, q8, sw, k, bias=b)
    assert_f32_close(host(y), ref, b)
    y2 = nat.w8a8_linear(dev(x), dev(q8), dev(sw), bias=dev(b), path=path)
    assert np.array_equal(host(y).view(np.uint32), host(y2).view(np.uint32))


@pytest.mark.parametrize("path", ["decode", "tc"])
def test_w8a8_largest_k_full_code_range(nat, path):
    """K = W8A8_MAX_K with every code at +127 on both sides: the accumulator
    127 * 127 * K is the largest that fits INT32 and must come out exact;
    alternating signs on another channel give 0."""
    k, n, m = 133144, 16, 2
    w = np.ones((k, n), np.float32)
    w[1::2, 1] = -1.0
    x = np.ones((m, k), np.float32)
    q8, sw = oracle.w8_quantize(w)
    acc = host(nat.w8a8_linear(dev(x), dev(q8), dev(sw), out="s32", path=path))
    assert acc[0, 0] == 127 * 127 * k and acc[0, 1] == 0
    assert np.array_equal(acc, oracle.linear8(x, q8, sw, k, out="s32"))


@pytest.mark.parametrize("m", synth.DECODE_MS)
def test_w8a8_decode_full_size(nat, m):
    """Decode shape K = N = 4096 at M = 1, 4, 16, auto dispatch, every output,
    with and without the static-weights promise."""
    c = synth.decode_case(m)
    q8, sw = oracle.w8_quantize(c.w)
    wqd, swd = nat.w8_quantize(dev(c.w))
    assert np.array_equal(host(wqd), q8)
    ref = oracle.linear8(c.x, q8, sw, synth.DECODE_K, out="s32")
    for static in (False, True):
        acc = nat.w8a8_linear(dev(c.x), wqd, swd, out="s32", static_weights=static)
        assert nat.last_kernel() == "k_linear8_decode"
        assert np.array_equal(host(acc), ref)


def test_w8a8_prefill_full_size_sampled(nat):
    """Prefill shape M = 2048, K = 4096, N = 11008 on the tensor cores; the
    oracle recomputes sampled rows x channels (each row quantized over its
    full K) and the INT32 accumulators of the sample match bit for bit."""
    c = synth.prefill_case()
    k = c.w.shape[0]
    wqd, swd = nat.w8_quantize(dev(c.w))
    rng = synth.rng_for(2400, 0)
    rows = np.sort(rng.choice(c.x.shape[0], 24, replace=False))
    cols = np.sort(rng.choice(c.w.shape[1], 96, replace=False))
    q8_s, sw_s = oracle.w8_quantize(c.w[:, cols])
    assert np.array_equal(host(wqd)[cols], q8_s)
    acc = host(nat.w8a8_linear(dev(c.x), wqd, swd, out="s32"))
    assert nat.last_kernel() == "k_gemm_tc"
    assert np.array_equal(acc[np.ix_(rows, cols)], oracle.linear8(c.x[rows], q8_s, sw_s, k, out="s32"))
    y = host(nat.w8a8_linear(dev(c.x), wqd, swd, relu=True))
    assert_f32_close(y[np.ix_(rows, cols)], oracle.linear8(c.x[rows], q8_s, sw_s, k, relu=True))


@pytest.mark.parametrize("m,k,n", [(1024, 520, 4096), (2048, 777, 11008), (333, 1040, 2000)])
def test_w8a8_tc_token_tiles_sampled(nat, m, k, n):
    """Shapes on which the tensor-core GEMM's tile estimate picks each of its
    W8A8 token tiles (128, 160, and 64 with a ragged last tile): sampled
    rows x channels, INT32 bit for bit."""
    x, w, _ = _case(m, k, n, seed=2500 + m)
    wqd, swd = nat.w8_quantize(dev(w))
    rng = synth.rng_for(2500, m)
    rows = np.sort(rng.choice(m, 20, replace=False))
    rows[-1] = m - 1  # the last row of the last (ragged) token tile
    cols = np.sort(rng.choice(n, 80, replace=False))
    q8_s, sw_s = oracle.w8_quantize(w[:, cols])
    acc = host(nat.w8a8_linear(dev(x), wqd, swd, out="s32", path="tc"))
    assert np.array_equal(acc[np.ix_(rows, cols)], oracle.linear8(x[rows], q8_s, sw_s, k, out="s32"))
