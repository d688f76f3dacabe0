"""GPU parity of the cluster K-split decode kernel (k_decode_split) and of the
layer-chaining entry point (w4a8_linear_chain) against the CPU oracle.

Bars: the INT32 accumulators bit-exact; float32 and bf16 outputs bit-exact as
well, because these kernels dequantize with the oracle's own float32
operations (one multiply sx * sw, one IEEE division, the bias add, the ReLU
select) - a stronger bar than the layer's 1e-6 relative.
"""
import numpy as np
import pytest
import torch

import oracle
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


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def host(t):
    torch.cuda.synchronize()
    return t.cpu().numpy()


def bits(a):
    a = np.asarray(a)
    return a.view(np.uint16 if a.dtype == np.uint16 or a.itemsize == 2 else np.uint32)


def _case(m, k, n, seed, outliers=4):
    w = synth.linear_weights(k, n, 0.02, seed)
    x, _ = synth.linear_activations(m, k, seed, outlier_count=min(outliers, k), outlier_factor=20.0)
    b = synth.bias_vector(n, seed)
    return x, w, b


def _parts(y):
    """Per-row abs-max over every 16 consecutive columns (the chaining parts)."""
    m, n = y.shape
    p = -(-n // 16)
    pad = np.zeros((m, 16 * p), np.float32)
    pad[:, :n] = np.abs(y)
    return pad.reshape(m, p, 16).max(axis=2)


# K slices: 1 chunk (K <= 128), odd K, a ragged last slice, clusters of 1..8
# CTAs with 1..8 chunks each; N tails inside a warp's 16 channels and a CTA's
# 128; M on both sides of the 8-token tile.
SHAPES = [(1, 64, 16), (1, 4096, 4096), (2, 33, 17), (3, 1152, 256), (5, 1001, 130), (8, 256, 40),
          (9, 6912, 1152), (12, 520, 72), (16, 4096, 64), (16, 8192, 200), (16, 7, 300), (4, 129, 1000),
          (7, 2000, 129)]


@pytest.mark.parametrize("m,k,n", SHAPES)
def test_split_bit_exact_f32_and_int8_input(nat, m, k, n):
    x, w, _ = _case(m, k, n, seed=2000 + m + k + n)
    wp, sw = oracle.w4_quantize_pack(w)
    xd, wpd, swd = dev(x), dev(wp), dev(sw)
    acc_ref = oracle.linear(x, wp, sw, k, out="s32")
    y_ref = oracle.linear(x, wp, sw, k)
    # float32 input: the kernel quantizes its slices itself (one launch)
    acc = nat.w4a8_linear(xd, wpd, swd, out="s32", path="split")
    assert nat.last_kernel() == "k_decode_split" and nat.last_launch_count() == 1
    assert np.array_equal(host(acc), acc_ref)
    y = nat.w4a8_linear(xd, wpd, swd, path="split")
    assert np.array_equal(bits(host(y)), bits(y_ref))
    # INT8 input
    xq, sx = nat.a8_quantize_rows(xd)
    accq = nat.w4a8_linear_q(xq, sx, k, wpd, swd, out="s32", path="split")
    assert nat.last_kernel() == "k_decode_split"
    assert np.array_equal(host(accq), acc_ref)
    yq = nat.w4a8_linear_q(xq, sx, k, wpd, swd, path="split")
    assert np.array_equal(bits(host(yq)), bits(y_ref))


@pytest.mark.parametrize("relu", [False, True])
@pytest.mark.parametrize("with_bias", [False, True])
@pytest.mark.parametrize("static", [False, True])
def test_split_epilogue_forms(nat, relu, with_bias, static):
    m, k, n = 11, 1500, 200
    x, w, b = _case(m, k, n, seed=2100 + relu + 2 * with_bias)
    x[3] = 0.0                                   # an all-zero row: scale 1, output = bias
    bias = b if with_bias else None
    wp, sw = oracle.w4_quantize_pack(w)
    args = (dev(x), dev(wp), dev(sw))
    torch.cuda.synchronize()
    bd = None if bias is None else dev(bias)
    y = nat.w4a8_linear(*args, bias=bd, relu=relu, path="split", static_weights=static)
    ref = oracle.linear(x, wp, sw, k, bias=bias, relu=relu)
    assert np.array_equal(bits(host(y)), bits(ref))
    yb = nat.w4a8_linear(*args, bias=bd, relu=relu, out="bf16", path="split", static_weights=static)
    refb = oracle.linear(x, wp, sw, k, bias=bias, relu=relu, out="bf16")
    assert np.array_equal(host(yb.view(torch.int16)).view(np.uint16), refb)


def test_split_ignores_int8_pad_bytes_and_keeps_canaries(nat):
    m, k, n = 6, 100, 24
    x, w, _ = _case(m, k, n, seed=2200)
    wp, sw = oracle.w4_quantize_pack(w)
    xq_ref, sx_ref = oracle.a8_quantize_rows(x, ldq=112)
    xq_dirty = xq_ref.copy()
    xq_dirty[:, k:] = 77                         # garbage past K meets zero nibbles
    ybuf = torch.full((m + 1, 32), 12345.0, device="cuda")
    y = ybuf[:m, :n]
    nat.w4a8_linear_q(dev(xq_dirty), dev(sx_ref), k, dev(wp), dev(sw), y=y, path="split")
    yb = host(ybuf)
    assert (yb[:m, n:] == 12345.0).all() and (yb[m:] == 12345.0).all()
    assert np.array_equal(bits(yb[:m, :n]), bits(oracle.linear_q(xq_ref, sx_ref, wp, sw, k)))


def test_split_rejects_shapes_it_cannot_run(nat):
    for m, k in ((17, 64), (4, 8193)):           # more rows than a tile, more k than 8 x 8 chunks
        x = torch.zeros((m, k), device="cuda")
        wp = torch.zeros((16, nat.packed_ld(k)), dtype=torch.uint8, device="cuda")
        sw = torch.ones(16, device="cuda")
        with pytest.raises(nat.W4A8Error) as e:
            nat.w4a8_linear(x, wp, sw, path="split")
        assert e.value.status == nat.ERR_UNSUPPORTED


def test_decode_kernels_agree_bit_for_bit(nat):
    """The three decode kernels, forced on the same shapes, give the same
    INT32 accumulators and float32 bits as the oracle."""
    for m, k, n in ((1, 4096, 512), (4, 1152, 256), (8, 2000, 130)):
        x, w, _ = _case(m, k, n, seed=2300 + m)
        wp, sw = oracle.w4_quantize_pack(w)
        xd, wpd, swd = dev(x), dev(wp), dev(sw)
        ref = oracle.linear(x, wp, sw, k, out="s32")
        yref = oracle.linear(x, wp, sw, k)
        for path, kernel in (("split", "k_decode_split"), ("ring", "k_decode_ring"), ("regs", "k_linear_decode")):
            acc = nat.w4a8_linear(xd, wpd, swd, out="s32", path=path)
            assert nat.last_kernel() == kernel
            assert np.array_equal(host(acc), ref), path
            y = nat.w4a8_linear(xd, wpd, swd, path=path)
            assert np.array_equal(bits(host(y)), bits(yref)), path


# ------------------------------------------------------ layer chaining ---

def test_chain_minimal_mlp(nat):
    """The page's model, Dense(10->32, ReLU) -> Dense(32->1), chained: the
    first layer's epilogue emits the row abs-max parts of its output, the
    second layer quantizes its rows from them inside its product kernel. One
    launch per layer (four without chaining), and the oracle's bits."""
    d = synth.minimal_mlp(seed=0)
    wp1, sw1 = nat.w4_quantize_pack(dev(d.w1))
    wp2, sw2 = nat.w4_quantize_pack(dev(d.w2))
    h, a1 = nat.w4a8_linear_chain(dev(d.x), wp1, sw1, bias=dev(d.b1), relu=True)
    assert nat.last_launch_count() == 1
    y, a2 = nat.w4a8_linear_chain(h, wp2, sw2, x_amax=a1, bias=dev(d.b2))
    assert nat.last_launch_count() == 1
    wp1r, sw1r = oracle.w4_quantize_pack(d.w1)
    h_ref = oracle.linear(d.x, wp1r, sw1r, 10, bias=d.b1, relu=True)
    assert np.array_equal(bits(host(h)), bits(h_ref))
    assert np.array_equal(bits(host(a1)), bits(_parts(h_ref)))
    ref = oracle.mlp(d.x, d.w1, d.b1, d.w2, d.b2)
    assert np.array_equal(bits(host(y)), bits(ref))
    assert np.array_equal(bits(host(a2)), bits(_parts(ref)))


@pytest.mark.parametrize("m", [1, 4, 16])
def test_chain_shared_input_projections(nat, m):
    """A Gemma3-1B-shaped block at decode: the o projection (1024 -> 1152)
    emits the parts of its output H; q, k, v (1152 -> 1024, 256, 256) and
    gate, up (1152 -> 6912) all read H and quantize it from those parts inside
    their own kernels (one launch each, no activation pass). Their outputs
    hold the oracle's bits for layers fed with H."""
    x = synth.gemma_activations(m, 1024, sub=3)
    wo = synth.gemma_weights(0, 3)
    wpo, swo = oracle.w4_quantize_pack(wo)
    h, a = nat.w4a8_linear_chain(dev(x), dev(wpo), dev(swo))
    assert nat.last_launch_count() == 1
    h_host = host(h)
    h_ref = oracle.linear(x, wpo, swo, 1024)
    assert np.array_equal(bits(h_host), bits(h_ref))
    assert np.array_equal(bits(host(a)), bits(_parts(h_ref)))
    for p in (0, 1, 2, 4, 5):
        w = synth.gemma_weights(0, p)
        wp, sw = oracle.w4_quantize_pack(w)
        y, _ = nat.w4a8_linear_chain(h, dev(wp), dev(sw), x_amax=a, emit_amax=False)
        assert nat.last_launch_count() == 1 and nat.last_kernel() == "k_decode_split"
        assert np.array_equal(bits(host(y)), bits(oracle.linear(h_ref, wp, sw, 1152)))


@pytest.mark.parametrize("path", ["tc", "ring", "regs", "generic", "split"])
def test_chain_on_every_path(nat, path):
    """Chaining through every product path: the parts equal the output's
    row-chunk maxima and a consumer fed with them gives w4a8_linear's bits."""
    m = 40 if path in ("tc", "generic") else 6
    k1, n1, n2 = 600, 272, 96
    x, w1, b1 = _case(m, k1, n1, seed=2400)
    w2 = synth.linear_weights(n1, n2, 0.02, seed=2401)
    wp1, sw1 = oracle.w4_quantize_pack(w1)
    wp2, sw2 = oracle.w4_quantize_pack(w2)
    h, a = nat.w4a8_linear_chain(dev(x), dev(wp1), dev(sw1), bias=dev(b1), relu=True, path=path)
    h_ref = oracle.linear(x, wp1, sw1, k1, bias=b1, relu=True)
    hh = host(h)
    if path in ("tc",):
        assert (np.abs(hh - h_ref) <= 1e-6 * (np.abs(h_ref) + np.abs(b1)[None, :])).all()
    else:
        assert np.array_equal(bits(hh), bits(h_ref))
    assert np.array_equal(bits(host(a)), bits(_parts(hh)))
    y, _ = nat.w4a8_linear_chain(h, dev(wp2), dev(sw2), x_amax=a, emit_amax=False, path=path)
    y_plain = nat.w4a8_linear(h, dev(wp2), dev(sw2), path=path)
    assert np.array_equal(bits(host(y)), bits(host(y_plain)))
