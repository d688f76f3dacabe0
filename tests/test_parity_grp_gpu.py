"""GPU parity of the group-wise INT4 layer ("INT4" concept page, section 4.2:
every group of 128 weights along K has its own scale and zero point) against
the CPU oracle.

Bars: codes, scales and zero points bit-exact. The output is a float32 sum of
per-group terms that the kernel adds in another order than the oracle's loop.
Each side is within (2 ng + 2) * 2^-24 * sum_g |term_g| (+ 2^-24 |bias|) of
the exact sum, so the two agree within twice that (the bound is pinned
against float64 in the oracle tests). bfloat16 outputs within 1 ulp.
"""
import numpy as np
import pytest
import torch

import oracle
from tests.test_parity_gpu import dev, host
from w4a8_quantized_gemm_channel_b200 import synth

pytestmark = pytest.mark.gpu

GROUP = 128


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
    """The library's storage of the oracle's unsigned codes (q - 8, pad 0)."""
    n, ldp = wp_oracle.shape
    codes = np.zeros((n, 2 * ldp), np.int64)
    codes[:, 0::2], codes[:, 1::2] = wp_oracle & 0x0F, wp_oracle >> 4
    nib = np.zeros_like(codes)
    nib[:, :k] = (codes[:, :k] - 8) & 0xF
    return (nib[:, 0::2] | (nib[:, 1::2] << 4)).astype(np.uint8)


def _bound(x, wp, sa, zp, k, bias=None):
    """Twice the float32 summation bound around the exact group sum."""
    _, acc = oracle.linear_g(x, wp, sa, zp, k, GROUP, partials=True)
    _, sx = oracle.a8_quantize_rows(x)
    ng = sa.shape[1]
    terms = acc.astype(np.float64) / (sx.astype(np.float64)[:, None, None] * sa.astype(np.float64)[None, :, :])
    b = 0.0 if bias is None else np.abs(bias.astype(np.float64))[None, :]
    return 2 * ((2 * ng + 2) * 2.0 ** -24 * np.abs(terms).sum(axis=2) + 2.0 ** -24 * b) + 1e-30


@pytest.mark.parametrize("k,n", [(1, 1), (130, 40), (300, 33), (4096, 96)])
def test_w4g_quantize_pack_bit_exact(nat, k, n):
    w = synth.linear_weights(k, n, 0.02, seed=4000 + k + n)
    if n > 3 and k > 1:
        w[: min(k, GROUP), 2] = 0.125  # a constant group
    wp, sa, zp = oracle.w4g_quantize_pack(w, GROUP)
    wpd, sad, zpd = nat.w4g_quantize_pack(dev(w))
    assert np.array_equal(host(sad).view(np.uint32), sa.view(np.uint32))
    assert np.array_equal(host(zpd), zp)
    assert np.array_equal(host(wpd), _stored_bytes(wp, k))


@pytest.mark.parametrize("m,k,n", [(1, 130, 40), (3, 300, 17), (8, 1000, 64), (16, 4096, 96), (40, 256, 33),
                                   (17, 129, 20)])
@pytest.mark.parametrize("bias_relu", [False, True])
def test_w4g_linear_within_bound(nat, m, k, n, bias_relu):
    x, w, b = _case(m, k, n, seed=4100 + m + k)
    wp, sa, zp = oracle.w4g_quantize_pack(w, GROUP)
    wpd, sad, zpd = nat.w4g_quantize_pack(dev(w))
    bias = b if bias_relu else None
    y = host(nat.w4g_linear(dev(x), wpd, sad, zpd, bias=None if bias is None else dev(bias), relu=bias_relu))
    assert nat.last_kernel() == "k_linear_g" and nat.last_launch_count() == 2
    ref = oracle.linear_g(x, wp, sa, zp, k, GROUP, bias=bias, relu=bias_relu)
    assert (np.abs(y.astype(np.float64) - ref) <= _bound(x, wp, sa, zp, k, bias)).all()
    yb = nat.w4g_linear(dev(x), wpd, sad, zpd, bias=None if bias is None else dev(bias), relu=bias_relu,
                        out="bf16")
    a = host(yb.view(torch.int16)).view(np.int16).astype(np.int32)
    r = oracle.to_bf16_bits(ref).view(np.int16).astype(np.int32)
    assert (np.abs(a - r) <= 1).all()


def test_w4g_q_ignores_activation_pad_bytes_and_static_weights(nat):
    """INT8 rows with a stride past K (K not a multiple of 16) and garbage pad
    bytes: the group row sums stop at K; the static-weights promise gives the
    same bits."""
    m, k, n = 12, 300, 48
    x, w, b = _case(m, k, n, seed=4200)
    wp, sa, zp = oracle.w4g_quantize_pack(w, GROUP)
    wpd, sad, zpd = nat.w4g_quantize_pack(dev(w))
    xq, sx = oracle.a8_quantize_rows(x, ldq=320)
    xq[:, k:] = 101
    y = host(nat.w4g_linear_q(dev(xq), dev(sx), k, wpd, sad, zpd, bias=dev(b)))
    ref = oracle.linear_g(x, wp, sa, zp, k, GROUP, bias=b)
    assert (np.abs(y.astype(np.float64) - ref) <= _bound(x, wp, sa, zp, k, b)).all()
    y2 = host(nat.w4g_linear_q(dev(xq), dev(sx), k, wpd, sad, zpd, bias=dev(b), static_weights=True))
    assert np.array_equal(y.view(np.uint32), y2.view(np.uint32))
