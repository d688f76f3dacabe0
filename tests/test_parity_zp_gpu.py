"""GPU parity of the zero-point INT4 layer (asymmetric per-channel weights:
the "INT4" concept page, section 4.1, and the "4-bit Integer Quantization for
LLMs" page, section "Weight quantization") against the CPU oracle.

Bars as for the W4A8 layer: codes, scales, zero points and the INT32
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


def _case(m, k, n, seed):
    w = synth.linear_weights(k, n, 0.02, seed)
    x, _ = synth.linear_activations(m, k, seed, outlier_count=min(4, k), outlier_factor=20.0)
    b = synth.bias_vector(n, seed)
    return x, w, b


def _stored_bytes(wp_oracle, k):
    """The library's storage of the oracle's unsigned codes: each code as the
    signed nibble q - 8, pad nibbles 0 (built here from the nibbles)."""
    n, ldp = wp_oracle.shape
    codes = np.zeros((n, 2 * ldp), np.int64)
    codes[:, 0::2], codes[:, 1::2] = wp_oracle & 0x0F, wp_oracle >> 4
    nib = np.zeros_like(codes)
    nib[:, :k] = (codes[:, :k] - 8) & 0xF
    return (nib[:, 0::2] | (nib[:, 1::2] << 4)).astype(np.uint8)


@pytest.mark.parametrize("k,n", [(1, 1), (7, 33), (64, 130), (1153, 256), (4096, 96)])
def test_w4z_quantize_pack_bit_exact(nat, k, n):
    w = synth.linear_weights(k, n, 0.02, seed=3000 + k + n)
    if n > 5:
        w[:, 3] = 0.25        # a constant column: no range
        w[:, 5] = np.abs(w[:, 5]) + 1.0  # all positive: a negative zero point
    wp, sa, zp = oracle.w4z_quantize_pack(w)
    wpd, sad, zpd = nat.w4z_quantize_pack(dev(w))
    assert np.array_equal(host(sad).view(np.uint32), sa.view(np.uint32))
    assert np.array_equal(host(zpd), zp)
    assert np.array_equal(host(wpd), _stored_bytes(wp, k))


@pytest.mark.parametrize("path", PATHS)
@pytest.mark.parametrize("m,k,n", [(1, 64, 16), (3, 33, 17), (8, 256, 40), (16, 4096, 64), (17, 300, 33),
                                   (300, 520, 300), (256, 4096, 1024)])
def test_w4z_s32_bit_exact(nat, path, m, k, n):
    x, w, _ = _case(m, k, n, seed=3100 + m + k + n)
    if n > 2:
        w[:, 2] = np.abs(w[:, 2]) + 0.5  # a negative zero point
    wp, sa, zp = oracle.w4z_quantize_pack(w)
    wpd, sad, zpd = nat.w4z_quantize_pack(dev(w))
    acc = nat.w4z_linear(dev(x), wpd, sad, zpd, out="s32", path=path)
    # the activation pass (which writes the row sums too), then the product
    # with the zero-point correction in its epilogue
    assert nat.last_path() == path and nat.last_launch_count() == 2
    assert np.array_equal(host(acc), oracle.linear_z(x, wp, sa, zp, k, out="s32"))


@pytest.mark.parametrize("path", ["split", "ring", "regs"])
@pytest.mark.parametrize("m,k,n", [(1, 64, 16), (3, 1001, 130), (8, 4096, 64)])
def test_w4z_every_decode_kernel(nat, path, m, k, n):
    """The zero-point correction in the epilogue of each decode kernel: INT32
    bit-exact and float32 within the bar, with a bias and ReLU."""
    x, w, b = _case(m, k, n, seed=3150 + m + k)
    w[:, 1] = np.abs(w[:, 1]) + 0.5      # a negative zero point
    wp, sa, zp = oracle.w4z_quantize_pack(w)
    wpd, sad, zpd = nat.w4z_quantize_pack(dev(w))
    acc = nat.w4z_linear(dev(x), wpd, sad, zpd, out="s32", path=path)
    assert np.array_equal(host(acc), oracle.linear_z(x, wp, sa, zp, k, out="s32"))
    y = nat.w4z_linear(dev(x), wpd, sad, zpd, bias=dev(b), relu=True, path=path)
    assert_f32_close(host(y), oracle.linear_z(x, wp, sa, zp, k, bias=b, relu=True), b)


@pytest.mark.parametrize("path", PATHS)
@pytest.mark.parametrize("relu", [False, True])
def test_w4z_f32_bf16_bias_relu(nat, path, relu):
    m, k, n = 37, 700, 150
    x, w, b = _case(m, k, n, seed=3200)
    x[5] = 0.0
    wp, sa, zp = oracle.w4z_quantize_pack(w)
    wpd, sad, zpd = nat.w4z_quantize_pack(dev(w))
    bd = dev(b)
    y = nat.w4z_linear(dev(x), wpd, sad, zpd, bias=bd, relu=relu, path=path)
    assert_f32_close(host(y), oracle.linear_z(x, wp, sa, zp, k, bias=b, relu=relu), b)
    yb = nat.w4z_linear(dev(x), wpd, sad, zpd, bias=bd, relu=relu, out="bf16", path=path)
    assert_bf16_within_ulp(host(yb.view(torch.int16)), oracle.linear_z(x, wp, sa, zp, k, bias=b, relu=relu,
                                                                        out="bf16"))


@pytest.mark.parametrize("path", PATHS)
def test_w4z_q_ignores_activation_pad_bytes(nat, path):
    """INT8 rows with a stride past K and garbage pad bytes: the row sums stop at
    K and the pad multiplies zero nibbles; the same bits as w4z_linear."""
    m, k, n = 20, 100, 48
    x, w, b = _case(m, k, n, seed=3300)
    wp, sa, zp = oracle.w4z_quantize_pack(w)
    wpd, sad, zpd = nat.w4z_quantize_pack(dev(w))
    xq, sx = oracle.a8_quantize_rows(x, ldq=128)
    xq[:, k:] = -77
    y = nat.w4z_linear_q(dev(xq), dev(sx), k, wpd, sad, zpd, bias=dev(b), path=path)
    assert nat.last_launch_count() == 2
    assert_f32_close(host(y), oracle.linear_z(x, wp, sa, zp, k, bias=b), b)
    y2 = nat.w4z_linear(dev(x), wpd, sad, zpd, bias=dev(b), path=path)
    assert np.array_equal(host(y).view(np.uint32), host(y2).view(np.uint32))


@pytest.mark.parametrize("m", synth.DECODE_MS)
def test_w4z_decode_full_size(nat, m):
    """K = N = 4096 at M = 1, 4, 16, auto dispatch, every INT32 output, with
    and without the static-weights promise."""
    c = synth.decode_case(m)
    wp, sa, zp = oracle.w4z_quantize_pack(c.w)
    wpd, sad, zpd = nat.w4z_quantize_pack(dev(c.w))
    ref = oracle.linear_z(c.x, wp, sa, zp, synth.DECODE_K, out="s32")
    for static in (False, True):
        acc = nat.w4z_linear(dev(c.x), wpd, sad, zpd, out="s32", static_weights=static)
        assert np.array_equal(host(acc), ref)
