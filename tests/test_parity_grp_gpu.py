"""GPU parity of the group-wise INT4 layer ("INT4" concept page, section 4.2:
every group of 128 weights along K has its own scale and zero point) against
the CPU oracle.

Bars: codes, scales and zero points bit-exact. The output is a float32 sum of
per-group terms that the kernel adds in another order than the oracle's loop.
Each side is within (2 ng + 2) * 2^-24 * sum_g |term_g| (+ 2^-24 |bias|) of
the exact sum, so the two agree within twice that (the bound is pinned
against float64 in the oracle tests). bfloat16 outputs: that bound plus
the bf16 rounding of the value.
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


def _bf16_close(y_bf16_bits, ref, bound):
    """bfloat16 outputs of a float32 result within `bound` of the oracle's:
    |bf16(y) - ref| <= bound + 2^-8 (|ref| + bound) (bf16 keeps 8
    significant bits, so rounding to it moves a value by at most 2^-8 of
    it). A 1-ulp bar on the bits is not implied: an output
    within the bound of zero may be clipped by ReLU on one side only."""
    v = (np.asarray(y_bf16_bits).astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return (np.abs(v - ref) <= bound + 2.0 ** -8 * (np.abs(ref) + bound)).all()


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
    assert nat.last_kernel() == ("k_linear_g" if m <= 16 else "k_gemm_tc_grp") and nat.last_launch_count() == 2
    ref = oracle.linear_g(x, wp, sa, zp, k, GROUP, bias=bias, relu=bias_relu)
    assert (np.abs(y.astype(np.float64) - ref) <= _bound(x, wp, sa, zp, k, bias)).all()
    yb = nat.w4g_linear(dev(x), wpd, sad, zpd, bias=None if bias is None else dev(bias), relu=bias_relu,
                        out="bf16")
    assert _bf16_close(host(yb.view(torch.int16)).view(np.uint16), ref, _bound(x, wp, sa, zp, k, bias))


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


# ------------------------------------------------- tensor-core form ---

@pytest.mark.parametrize("m,k,n", [(200, 1000, 300), (129, 4096, 130), (300, 1153, 64), (3, 256, 40),
                                   (640, 128, 1000), (17, 100, 129)])
@pytest.mark.parametrize("bias_relu", [False, True])
def test_w4g_tensor_core_within_bound(nat, m, k, n, bias_relu):
    """The tensor-core form (tcgen05, a TMEM accumulator drained per group of
    128 k): groups that straddle pipeline stages, a ragged last group, token
    and channel tails, a single-group K; forced onto the tensor cores for few
    rows too. Within the group-sum bound of the oracle, bf16 within 1 ulp."""
    x, w, b = _case(m, k, n, seed=4300 + m + k)
    if n > 3:
        w[:, 2] = np.abs(w[:, 2]) + 0.3        # a negative zero point in every group
    wp, sa, zp = oracle.w4g_quantize_pack(w, GROUP)
    wpd, sad, zpd = nat.w4g_quantize_pack(dev(w))
    bias = b if bias_relu else None
    bd = None if bias is None else dev(bias)
    y = host(nat.w4g_linear(dev(x), wpd, sad, zpd, bias=bd, relu=bias_relu, path="tc"))
    assert nat.last_kernel() == "k_gemm_tc_grp" and nat.last_launch_count() == 2
    ref = oracle.linear_g(x, wp, sa, zp, k, GROUP, bias=bias, relu=bias_relu)
    assert (np.abs(y.astype(np.float64) - ref) <= _bound(x, wp, sa, zp, k, bias)).all()
    yb = nat.w4g_linear(dev(x), wpd, sad, zpd, bias=bd, relu=bias_relu, out="bf16", path="tc")
    assert _bf16_close(host(yb.view(torch.int16)).view(np.uint16), ref, _bound(x, wp, sa, zp, k, bias))


def test_w4g_tensor_core_int8_input_and_static_weights(nat):
    """INT8 rows in natural k order (w4g_linear_q) and the permuted layout of
    the activation pass give the same bits; so does the static-weights
    promise; garbage past K in the rows does not matter."""
    m, k, n = 70, 300, 160
    x, w, b = _case(m, k, n, seed=4400)
    wp, sa, zp = oracle.w4g_quantize_pack(w, GROUP)
    wpd, sad, zpd = nat.w4g_quantize_pack(dev(w))
    xq, sx = oracle.a8_quantize_rows(x, ldq=320)
    xq[:, k:] = -99
    y = host(nat.w4g_linear_q(dev(xq), dev(sx), k, wpd, sad, zpd, bias=dev(b)))
    assert nat.last_kernel() == "k_gemm_tc_grp"
    ref = oracle.linear_g(x, wp, sa, zp, k, GROUP, bias=b)
    assert (np.abs(y.astype(np.float64) - ref) <= _bound(x, wp, sa, zp, k, b)).all()
    torch.cuda.synchronize()
    y2 = host(nat.w4g_linear(dev(x), wpd, sad, zpd, bias=dev(b), static_weights=True))
    assert np.array_equal(y.view(np.uint32), y2.view(np.uint32))


def test_w4g_tensor_core_prefill_size_sampled(nat):
    """The prefill shape (M = 2048, K = 4096, N = 11008) in group-wise form:
    sampled rows x channels recomputed by the oracle (each channel's groups
    are quantized on their own, so a column sample of W gives the same codes,
    scales and zero points)."""
    c = synth.prefill_case()
    k, n = c.w.shape
    wpd, sad, zpd = nat.w4g_quantize_pack(dev(c.w))
    y = host(nat.w4g_linear(dev(c.x), wpd, sad, zpd))
    rng = synth.rng_for(44, 44)
    rows = np.unique(np.concatenate([[0, 2047], rng.integers(0, 2048, size=6)]))
    cols = np.unique(np.concatenate([[0, n - 1], rng.integers(0, n, size=40)]))
    wp, sa, zp = oracle.w4g_quantize_pack(np.ascontiguousarray(c.w[:, cols]), GROUP)
    assert np.array_equal(host(sad)[cols].view(np.uint32), sa.view(np.uint32))
    ref = oracle.linear_g(c.x[rows], wp, sa, zp, k, GROUP)
    bound = _bound(c.x[rows], wp, sa, zp, k)
    assert (np.abs(y[np.ix_(rows, cols)].astype(np.float64) - ref) <= bound).all()
