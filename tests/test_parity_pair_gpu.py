"""GPU parity of the two-SM tensor-core product (k_gemm_tc_pair, forced with
path "tc2") against the CPU oracle, and against the one-SM tensor-core kernel.

The pair kernel computes the same INT32 accumulator and runs the same
epilogue arithmetic as the one-SM kernel, so besides the oracle bars (INT32
bit-exact, float32 within 1e-6 relative, bfloat16 within 1 ulp) its float
and bf16 outputs must equal the one-SM kernel's bit for bit.

Shapes span several 256-channel x 192-token pair tiles, ragged tails in both
directions, K tails inside a 256-k stage, more tiles than resident pairs (the
persistent loop) and the zero-point epilogue.
"""
import numpy as np
import pytest
import torch

import oracle
from tests.test_parity_gpu import _case, _sampled_check, assert_bf16_within_ulp, assert_f32_close, dev, host
from w4a8_quantized_gemm_channel_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def nat():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from w4a8_quantized_gemm_channel_b200 import native
    native.get_device_status(clear=True)
    yield native
    assert native.get_device_status() == 0, "a kernel recorded an internal fault"


@pytest.mark.parametrize("m,k,n", [(17, 300, 33), (192, 256, 256), (193, 1000, 257), (300, 520, 300),
                                   (256, 4096, 1024), (385, 2049, 700)])
def test_pair_s32_bit_exact(nat, m, k, n):
    x, w, _ = _case(m, k, n, seed=7000 + m + k + n)
    wp, sw = oracle.w4_quantize_pack(w)
    acc = nat.w4a8_linear(dev(x), dev(wp), dev(sw), out="s32", path="tc2")
    assert nat.last_path() == "tc" and nat.last_kernel() == "k_gemm_tc_pair"
    assert np.array_equal(host(acc), oracle.linear(x, wp, sw, k, out="s32"))


@pytest.mark.parametrize("relu", [False, True])
@pytest.mark.parametrize("with_bias", [False, True])
def test_pair_epilogue_forms(nat, relu, with_bias):
    m, k, n = 230, 777, 300
    x, w, b = _case(m, k, n, seed=7100 + relu + 2 * with_bias)
    bias = b if with_bias else None
    wp, sw = oracle.w4_quantize_pack(w)
    args = (dev(x), dev(wp), dev(sw))
    bd = None if bias is None else dev(bias)
    for out in ("f32", "bf16"):
        y2 = nat.w4a8_linear(*args, bias=bd, relu=relu, out=out, path="tc2")
        assert nat.last_kernel() == "k_gemm_tc_pair"
        y1 = nat.w4a8_linear(*args, bias=bd, relu=relu, out=out, path="tc")
        assert nat.last_kernel() == "k_gemm_tc"
        h2 = host(y2.view(torch.int16) if out == "bf16" else y2)
        assert np.array_equal(h2, host(y1.view(torch.int16) if out == "bf16" else y1))
        ref = oracle.linear(x, wp, sw, k, bias=bias, relu=relu, out=out)
        if out == "bf16":
            assert_bf16_within_ulp(h2, ref)
        else:
            assert_f32_close(h2, ref, bias)


def test_pair_many_tiles_persistent_loop(nat):
    """More pair tiles than resident pairs: 11 token tiles x 8 channel tiles
    (88 > 74), so pairs take a second tile and reuse the double-buffered
    accumulator."""
    m, k, n = 2000, 512, 2000
    x, w, _ = _case(m, k, n, seed=7200)
    wp, sw = oracle.w4_quantize_pack(w)
    acc = nat.w4a8_linear(dev(x), dev(wp), dev(sw), out="s32", path="tc2")
    assert np.array_equal(host(acc), oracle.linear(x, wp, sw, k, out="s32"))
    y2 = nat.w4a8_linear(dev(x), dev(wp), dev(sw), path="tc2")
    y1 = nat.w4a8_linear(dev(x), dev(wp), dev(sw), path="tc")
    assert np.array_equal(host(y2), host(y1))


def test_pair_linear_q_natural_order_and_pad_bytes(nat):
    """The INT8-activation entry point feeds natural k order (the unpack with
    byte permutes); garbage past K in the activation rows must not matter."""
    m, k, n = 200, 300, 260
    x, w, _ = _case(m, k, n, seed=7300)
    wp, sw = oracle.w4_quantize_pack(w)
    xq_ref, sx_ref = oracle.a8_quantize_rows(x, ldq=320)
    xq_dirty = xq_ref.copy()
    xq_dirty[:, k:] = 77
    acc = nat.w4a8_linear_q(dev(xq_dirty), dev(sx_ref), k, dev(wp), dev(sw), out="s32", path="tc2")
    assert nat.last_kernel() == "k_gemm_tc_pair"
    assert np.array_equal(host(acc), oracle.linear_q(xq_ref, sx_ref, wp, sw, k, out="s32"))


@pytest.mark.parametrize("n,out", [(270, "f32"), (272, "f32"), (264, "bf16"), (270, "bf16"), (268, "s32")])
def test_pair_output_stride_leaves_canaries(nat, n, out):
    """Outputs past column N and past row M stay untouched, for row lengths
    that end on a 16-byte boundary (staged bulk stores) and that do not
    (direct stores)."""
    m, k = 197, 256
    x, w, _ = _case(m, k, n, seed=7400 + n)
    wp, sw = oracle.w4_quantize_pack(w)
    dt = {"f32": torch.float32, "bf16": torch.bfloat16, "s32": torch.int32}[out]
    ybuf = torch.full((m + 3, 288), 12345, dtype=dt, device="cuda")
    y = ybuf[:m, :n]
    nat.w4a8_linear(dev(x), dev(wp), dev(sw), y=y, out=out, path="tc2")
    yb = host(ybuf.float())
    fill = float(torch.tensor(12345, dtype=dt).float())     # the canary as the dtype holds it
    assert (yb[:m, n:] == fill).all() and (yb[m:] == fill).all()
    if out == "f32":
        assert_f32_close(yb[:m, :n], oracle.linear(x, wp, sw, k))
    elif out == "s32":
        assert np.array_equal(host(ybuf)[:m, :n], oracle.linear(x, wp, sw, k, out="s32"))
    else:
        assert_bf16_within_ulp(host(y.contiguous().view(torch.int16)), oracle.linear(x, wp, sw, k, out="bf16"))


def test_pair_zero_point_epilogue(nat):
    m, k, n = 300, 520, 300
    x, w, b = _case(m, k, n, seed=7500)
    w[:, 2] = np.abs(w[:, 2]) + 0.5  # a negative zero point
    wp, sa, zp = oracle.w4z_quantize_pack(w)
    wpd, sad, zpd = nat.w4z_quantize_pack(dev(w))
    acc = nat.w4z_linear(dev(x), wpd, sad, zpd, out="s32", path="tc2")
    assert nat.last_kernel() == "k_gemm_tc_pair"
    assert np.array_equal(host(acc), oracle.linear_z(x, wp, sa, zp, k, out="s32"))
    y = nat.w4z_linear(dev(x), wpd, sad, zpd, bias=dev(b), relu=True, path="tc2")
    assert_f32_close(host(y), oracle.linear_z(x, wp, sa, zp, k, bias=b, relu=True), b)


def test_pair_prefill_full_size_sampled(nat):
    """M = 2048, K = 4096, N = 11008 through the pair kernel; sampled rows x
    channels recomputed by the oracle."""
    c = synth.prefill_case()
    wpd, swd = nat.w4_quantize_pack(dev(c.w))
    rng = synth.rng_for(11, 11)
    rows = np.unique(np.concatenate([[0, 2047], rng.integers(0, 2048, size=6)]))
    cols = np.unique(np.concatenate([[0, 11007], rng.integers(0, 11008, size=60)]))
    _sampled_check(nat, c.x, c.w, wpd, swd, rows, cols, path="tc2")


def test_pair_rejects_other_forms(nat):
    """The pair kernel serves the INT4 codes in the 16 q form (K <= 131072)
    only: W8A8, group-wise and larger K are refused, not rerouted."""
    m, n = 20, 16
    x, w, _ = _case(m, 64, n, seed=7600)
    wq, sw8 = nat.w8_quantize(dev(w))
    with pytest.raises(nat.W4A8Error) as e:
        nat.w8a8_linear(dev(x), wq, sw8, path="tc2")
    assert e.value.status == nat.ERR_UNSUPPORTED
    wg, sag, zpg = nat.w4g_quantize_pack(dev(w))
    with pytest.raises(nat.W4A8Error) as e:
        nat.w4g_linear(dev(x), wg, sag, zpg, path="tc2")
    assert e.value.status == nat.ERR_UNSUPPORTED
    k = 131073
    xl = torch.zeros((m, k), device="cuda")
    wpl = torch.zeros((n, nat.packed_ld(k)), dtype=torch.uint8, device="cuda")
    swl = torch.ones(n, device="cuda")
    with pytest.raises(nat.W4A8Error) as e:
        nat.w4a8_linear(xl, wpl, swl, path="tc2")
    assert e.value.status == nat.ERR_UNSUPPORTED


@pytest.mark.parametrize("out", ["f32", "bf16", "s32"])
def test_pair_unaligned_output_takes_direct_stores(nat, out):
    """An output whose base or row stride is not 16-byte aligned cannot take
    the staged bulk-store epilogue; the direct-store form gives the same bits."""
    m, k, n = 200, 384, 300
    x, w, _ = _case(m, k, n, seed=7700)
    wp, sw = oracle.w4_quantize_pack(w)
    args = (dev(x), dev(wp), dev(sw))
    dt = {"f32": torch.float32, "bf16": torch.bfloat16, "s32": torch.int32}[out]
    ref = nat.w4a8_linear(*args, out=out, path="tc2")          # aligned: staged stores
    ldy = n + 1                                                 # odd stride
    buf = torch.zeros(m * ldy + 8, dtype=dt, device="cuda")
    y_stride = buf[:m * ldy].view(m, ldy)[:, :n]
    nat.w4a8_linear(*args, out=out, path="tc2", y=y_stride)
    y_base = buf[1:1 + m * ldy].view(m, ldy)[:, :n]             # base off 16-byte alignment
    nat.w4a8_linear(*args, out=out, path="tc2", y=y_base)
    as_bits = (lambda t: host(t.view(torch.int16))) if out == "bf16" else host
    assert np.array_equal(as_bits(y_base.contiguous()), as_bits(ref))
    buf.zero_()
    nat.w4a8_linear(*args, out=out, path="tc2", y=y_stride)
    assert np.array_equal(as_bits(y_stride.contiguous()), as_bits(ref))
    assert (host(buf[:m * ldy].view(m, ldy)[:, n:].float()) == 0).all()


def test_pair_static_weights_gives_same_bits(nat):
    m, k, n = 600, 1152, 520
    x, w, b = _case(m, k, n, seed=7800)
    wp, sw = oracle.w4_quantize_pack(w)
    args = (dev(x), dev(wp), dev(sw))
    y0 = nat.w4a8_linear(*args, bias=dev(b), path="tc2")
    y1 = nat.w4a8_linear(*args, bias=dev(b), path="tc2", static_weights=True)
    assert np.array_equal(host(y0), host(y1))
    assert_f32_close(host(y1), oracle.linear(x, wp, sw, k, bias=b), b)
