"""GPU parity: every kernel path against the CPU oracle on the same seeded inputs.

Bars (the layer's stated tolerances):
  * packed weights, weight scales, INT8 activations, activation scales and the
    INT32 accumulator: bit-exact;
  * float32 output: |y - y_oracle| <= 1e-6 * |y_oracle| (with a bias,
    1e-6 * (|y_oracle| + |b|), since a sum can cancel);
  * bfloat16 output: within 1 bf16 ulp of the oracle's bf16 rounding.
"""
import numpy as np
import pytest
import torch

import oracle
from w4a8_quantized_gemm_channel_b200 import synth

pytestmark = pytest.mark.gpu

RTOL = 1e-6


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


def assert_f32_close(y, ref, bias=None, rtol=RTOL):
    y = np.asarray(y, np.float64)
    ref = np.asarray(ref, np.float64)
    scale = np.abs(ref)
    if bias is not None:
        scale = scale + np.abs(np.asarray(bias, np.float64))[None, :]
    bad = np.abs(y - ref) > rtol * scale
    assert not bad.any(), f"{bad.sum()} of {bad.size} outputs outside {rtol} relative"


def assert_bf16_within_ulp(ybits, refbits):
    a = np.asarray(ybits).view(np.int16).astype(np.int32)
    b = np.asarray(refbits).view(np.int16).astype(np.int32)
    assert (np.abs(a - b) <= 1).all()


# ------------------------------------------------------------ weights ---

@pytest.mark.parametrize("k,n", [(1, 1), (10, 32), (32, 1), (33, 7), (130, 45), (1152, 256),
                                 (4096, 4096)])
def test_quantize_pack_bit_exact(nat, k, n):
    w = synth.linear_weights(k, n, 0.02, seed=100 + k + n)
    if n > 2:
        w[:, 1] = 0.0                      # an all-zero output channel
    wp, sw = nat.w4_quantize_pack(dev(w))
    wp_ref, sw_ref = oracle.w4_quantize_pack(w)
    assert np.array_equal(host(sw).view(np.uint32), sw_ref.view(np.uint32))
    assert np.array_equal(host(wp), wp_ref)


@pytest.mark.parametrize("k,n", [(1, 32), (257, 40), (600, 64), (4097, 96), (6912, 64), (12288, 32),
                                 (12289, 32), (8192, 36)])
def test_quantize_pack_panel_path_bit_exact(nat, k, n):
    """Shapes around the single-pass (cluster panel) form's limits: one slice,
    a partial 32-channel panel, a cluster whose last slice lies past K, the
    largest K it takes (12288) and the first it hands to the two-pass form."""
    w = synth.linear_weights(k, n, 0.02, seed=150 + k + n)
    w[:, 3] = 0.0                          # an all-zero output channel
    w[k // 2, 5] = 0.5                     # a column's maximum in the middle slice
    wp, sw = nat.w4_quantize_pack(dev(w))
    wp_ref, sw_ref = oracle.w4_quantize_pack(w)
    assert np.array_equal(host(sw).view(np.uint32), sw_ref.view(np.uint32))
    assert np.array_equal(host(wp), wp_ref)


def test_quantize_pack_wide_stride_and_padding(nat):
    k, n = 77, 20
    w = synth.linear_weights(k, 24, 0.02, seed=7)     # ldw = 24 > N
    wd = dev(w)[:, :n]
    ldp = 96                                         # more than ceil(77/2)
    wp = torch.full((n, ldp), 0xAB, dtype=torch.uint8, device="cuda")
    nat.w4_quantize_pack(wd, wp=wp)
    wp_ref, _ = oracle.w4_quantize_pack(np.ascontiguousarray(w[:, :n]), ldp=ldp)
    assert np.array_equal(host(wp), wp_ref)          # pad bytes overwritten with 0
    # a row stride much wider than the codes need, on a 16-byte aligned
    # layout (single-pass form): the bytes past the cluster's rows are zeroed
    k, n = 600, 40
    w = synth.linear_weights(k, 48, 0.02, seed=8)
    wd = dev(w)[:, :n]
    ldp = 1024
    wp = torch.full((n, ldp), 0xAB, dtype=torch.uint8, device="cuda")
    nat.w4_quantize_pack(wd, wp=wp)
    wp_ref, _ = oracle.w4_quantize_pack(np.ascontiguousarray(w[:, :n]), ldp=ldp)
    assert np.array_equal(host(wp), wp_ref)


# -------------------------------------------------------- activations ---

@pytest.mark.parametrize("m,k", [(1, 1), (32, 10), (3, 37), (16, 4096), (2048, 4096), (5, 6912)])
def test_act_quant_bit_exact(nat, m, k):
    x, _ = synth.linear_activations(m, k, seed=200 + m, outlier_count=min(8, k), outlier_factor=20.0)
    if m > 2:
        x[1] = 0.0                          # an all-zero row
    xq, sx = nat.a8_quantize_rows(dev(x))
    ldq = xq.shape[1]
    xq_ref, sx_ref = oracle.a8_quantize_rows(x, ldq=ldq)
    assert np.array_equal(host(sx).view(np.uint32), sx_ref.view(np.uint32))
    assert np.array_equal(host(xq), xq_ref)


def test_act_quant_unaligned_stride(nat):
    x = synth.normal((9, 51), 1.0, synth.rng_for(3, 3))   # ldx = 51: no float4 loads
    xd = dev(x)[:, 1:50]
    xq, sx = nat.a8_quantize_rows(xd)
    xq_ref, sx_ref = oracle.a8_quantize_rows(np.ascontiguousarray(x[:, 1:50]), ldq=xq.shape[1])
    assert np.array_equal(host(xq), xq_ref)
    assert np.array_equal(host(sx), sx_ref)


def test_act_quant_empty(nat):
    x = torch.empty((0, 64), device="cuda")
    xq, sx = nat.a8_quantize_rows(x)
    assert xq.shape[0] == 0 and sx.shape[0] == 0


# ------------------------------------------------------------- linear ---

PATHS = ["generic", "decode", "tc"]


def _case(m, k, n, seed, outliers=4):
    w = synth.linear_weights(k, n, 0.02, seed)
    x, _ = synth.linear_activations(m, k, seed, outlier_count=min(outliers, k), outlier_factor=20.0)
    b = synth.bias_vector(n, seed)
    return x, w, b


@pytest.mark.parametrize("path", PATHS)
@pytest.mark.parametrize("m,k,n", [(1, 64, 16), (3, 33, 17), (8, 256, 40), (16, 4096, 64),
                                   (17, 300, 33), (40, 1000, 130), (300, 520, 300),
                                   (256, 4096, 1024)])
def test_linear_s32_bit_exact(nat, path, m, k, n):
    x, w, _ = _case(m, k, n, seed=300 + m + k + n)
    wp, sw = oracle.w4_quantize_pack(w)
    acc = nat.w4a8_linear(dev(x), dev(wp), dev(sw), out="s32", path=path)
    assert nat.last_path() == path
    assert np.array_equal(host(acc), oracle.linear(x, wp, sw, k, out="s32"))


@pytest.mark.parametrize("path", PATHS)
@pytest.mark.parametrize("relu", [False, True])
@pytest.mark.parametrize("with_bias", [False, True])
def test_linear_f32_and_bf16(nat, path, relu, with_bias):
    m, k, n = 12, 520, 72
    x, w, b = _case(m, k, n, seed=400 + relu + 2 * with_bias)
    bias = b if with_bias else None
    wp, sw = oracle.w4_quantize_pack(w)
    args = (dev(x), dev(wp), dev(sw))
    y = nat.w4a8_linear(*args, bias=None if bias is None else dev(bias), relu=relu, path=path)
    ref = oracle.linear(x, wp, sw, k, bias=bias, relu=relu)
    assert_f32_close(host(y), ref, bias)
    if relu:
        assert (host(y) >= 0).all()
    yb = nat.w4a8_linear(*args, bias=None if bias is None else dev(bias), relu=relu,
                         out="bf16", path=path)
    refb = oracle.linear(x, wp, sw, k, bias=bias, relu=relu, out="bf16")
    assert_bf16_within_ulp(host(yb.view(torch.int16)), refb)


@pytest.mark.parametrize("path", PATHS)
def test_linear_q_matches_oracle_and_ignores_pad_bytes(nat, path):
    m, k, n = 6, 100, 24
    x, w, _ = _case(m, k, n, seed=500)
    wp, sw = oracle.w4_quantize_pack(w)
    xq_ref, sx_ref = oracle.a8_quantize_rows(x, ldq=112)
    xq_dirty = xq_ref.copy()
    xq_dirty[:, k:] = 77                      # garbage past K must not matter
    y = nat.w4a8_linear_q(dev(xq_dirty), dev(sx_ref), k, dev(wp), dev(sw), path=path)
    assert_f32_close(host(y), oracle.linear_q(xq_ref, sx_ref, wp, sw, k))


@pytest.mark.parametrize("path", PATHS)
def test_linear_output_stride_leaves_canaries(nat, path):
    m, k, n = 5, 128, 20
    x, w, _ = _case(m, k, n, seed=600)
    wp, sw = oracle.w4_quantize_pack(w)
    ybuf = torch.full((m + 1, 32), 12345.0, device="cuda")
    y = ybuf[:m, :n]
    nat.w4a8_linear(dev(x), dev(wp), dev(sw), y=y, path=path)
    yb = host(ybuf)
    assert (yb[:m, n:] == 12345.0).all() and (yb[m:] == 12345.0).all()
    assert_f32_close(yb[:m, :n], oracle.linear(x, wp, sw, k))


def test_linear_zero_rows_is_a_noop(nat):
    wp = torch.zeros((8, 16), dtype=torch.uint8, device="cuda")
    sw = torch.ones(8, device="cuda")
    y = nat.w4a8_linear(torch.empty((0, 20), device="cuda"), wp, sw)
    assert y.shape == (0, 8)


def test_linear_zero_weight_column_gives_bias(nat):
    m, k, n = 4, 64, 8
    x, w, b = _case(m, k, n, seed=700)
    w[:, 3] = 0.0
    wpd, swd = nat.w4_quantize_pack(dev(w))
    y = host(nat.w4a8_linear(dev(x), wpd, swd, bias=dev(b)))
    assert (y[:, 3] == b[3]).all()


# ------------------------------------------------- the minimal model ---

def test_minimal_mlp_end_to_end(nat):
    """The page's model: Dense(10->32, ReLU) -> Dense(32->1), both W4A8."""
    d = synth.minimal_mlp(seed=0)
    wp1, sw1 = nat.w4_quantize_pack(dev(d.w1))
    wp2, sw2 = nat.w4_quantize_pack(dev(d.w2))
    h = nat.w4a8_linear(dev(d.x), wp1, sw1, bias=dev(d.b1), relu=True)
    y = host(nat.w4a8_linear(h, wp2, sw2, bias=dev(d.b2)))
    ref = oracle.mlp(d.x, d.w1, d.b1, d.w2, d.b2)
    assert np.array_equal(host(wp1), oracle.w4_quantize_pack(d.w1)[0])
    assert_f32_close(y, ref)
    x64 = d.x.astype(np.float64)
    yfp = np.maximum(x64 @ d.w1 + d.b1, 0) @ d.w2 + d.b2
    mse = float(np.mean((yfp - y) ** 2))
    assert 0 < mse <= 1e-2


def test_determinism(nat):
    m, k, n = 16, 4096, 512
    x, w, _ = _case(m, k, n, seed=800)
    wpd, swd = nat.w4_quantize_pack(dev(w))
    xd = dev(x)
    a = host(nat.w4a8_linear(xd, wpd, swd))
    b = host(nat.w4a8_linear(xd, wpd, swd))
    assert np.array_equal(a.view(np.uint32), b.view(np.uint32))


# --------------------------------------------- full-size workloads ---

@pytest.mark.parametrize("m", synth.DECODE_MS)
def test_decode_full_size(nat, m):
    """Decode single linear at full size (K = N = 4096), auto dispatch - the
    configuration the benchmark times - checked on every output."""
    c = synth.decode_case(m)
    wpd, swd = nat.w4_quantize_pack(dev(c.w))
    wp, sw = oracle.w4_quantize_pack(c.w)
    assert np.array_equal(host(wpd), wp)
    y = nat.w4a8_linear(dev(c.x), wpd, swd)
    assert_f32_close(host(y), oracle.linear(c.x, wp, sw, synth.DECODE_K))
    acc = nat.w4a8_linear(dev(c.x), wpd, swd, out="s32")
    assert np.array_equal(host(acc), oracle.linear(c.x, wp, sw, synth.DECODE_K, out="s32"))


@pytest.mark.parametrize("m,k,groups_over_2sm,kernel", [
    (1, 4096, -40, "k_decode_ring"), (2, 4096, -40, "k_decode_ring"), (3, 4096, -40, "k_linear_decode"),
    (8, 4096, -290, "k_linear_decode"), (8, 4097, -290, "k_decode_ring"), (8, 4096, 0, "k_linear_decode"),
    (8, 4096, 1, "k_decode_ring"), (16, 4096, -40, "k_linear_decode")])
def test_decode_kernel_choice_and_bits(nat, m, k, groups_over_2sm, kernel):
    """Few-row products with INT8 input on both sides of the rule that hands
    short layers (at most two 16-channel groups per SM) with K <= 4096 and
    M >= 3 to the register-path kernel: the kernel named, and the INT32
    accumulators bit for bit, with and without the static-weights promise."""
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    n = 16 * (2 * sms + groups_over_2sm)
    x, w, _ = _case(m, k, n, seed=1300 + m + k)
    wp, sw = oracle.w4_quantize_pack(w)
    ref = oracle.linear(x, wp, sw, k, out="s32")
    xq, sx = nat.a8_quantize_rows(dev(x))
    for static in (False, True):
        acc = nat.w4a8_linear_q(xq, sx, k, dev(wp), dev(sw), out="s32", static_weights=static)
        assert nat.last_kernel() == kernel
        assert np.array_equal(host(acc), ref)


def _sampled_check(nat, x, w, wpd, swd, rows, cols, relu=False, path="auto"):
    """Full-size run on the GPU; the oracle recomputes sampled rows x channels
    (each sampled row is quantized over its full K)."""
    wp_ref, sw_ref = oracle.w4_quantize_pack(w[:, cols]) if w is not None else (None, None)
    y = host(nat.w4a8_linear(dev(x), wpd, swd, relu=relu, path=path))
    wp_s = host(wpd)[cols]
    sw_s = host(swd)[cols]
    if wp_ref is not None:
        assert np.array_equal(wp_s, wp_ref)
        assert np.array_equal(sw_s, sw_ref)
    ref = oracle.linear(x[rows], wp_s, sw_s, x.shape[1], relu=relu)
    assert_f32_close(y[np.ix_(rows, cols)], ref)
    return y


def test_gemma_stack_shapes_sampled(nat):
    """One layer of the Gemma3-1B-shaped stack at M = 1 and M = 512."""
    rng = synth.rng_for(9, 9)
    for p, (name, k, n) in enumerate(synth.GEMMA_PROJ):
        w = synth.gemma_weights(0, p)
        wpd, swd = nat.w4_quantize_pack(dev(w))
        for m in synth.GEMMA_MS:
            x = synth.gemma_activations(m, k, sub=p)
            rows = np.unique(rng.integers(0, m, size=min(m, 8)))
            cols = np.unique(rng.integers(0, n, size=48))
            _sampled_check(nat, x, w, wpd, swd, rows, cols)


@pytest.mark.parametrize("path", ["tc", "auto"])
def test_prefill_full_size_int32_and_bf16_sampled(nat, path):
    """M = 2048, K = 4096, N = 11008 with INT32 and bf16 outputs, through the
    one-SM kernel (forced "tc") and the kernel the library picks (the CTA
    pair at this shape): sampled rows x channels against the oracle, INT32
    bit-exact and bf16 within 1 ulp."""
    c = synth.prefill_case()
    wpd, swd = nat.w4_quantize_pack(dev(c.w))
    rng = synth.rng_for(12, 12)
    rows = np.unique(np.concatenate([[0, 1, 2047], rng.integers(0, 2048, size=8)]))
    cols = np.unique(np.concatenate([[0, 255, 256, 11007], rng.integers(0, 11008, size=60)]))
    wp_s = host(wpd)[cols]
    sw_s = host(swd)[cols]
    acc = host(nat.w4a8_linear(dev(c.x), wpd, swd, out="s32", path=path))
    assert nat.last_kernel() == ("k_gemm_tc" if path == "tc" else "k_gemm_tc_pair")
    assert np.array_equal(acc[np.ix_(rows, cols)], oracle.linear(c.x[rows], wp_s, sw_s, c.x.shape[1], out="s32"))
    yb = host(nat.w4a8_linear(dev(c.x), wpd, swd, out="bf16", relu=True, path=path).view(torch.int16))
    ref = oracle.linear(c.x[rows], wp_s, sw_s, c.x.shape[1], relu=True, out="bf16")
    assert_bf16_within_ulp(yb[np.ix_(rows, cols)], ref)


def test_prefill_full_size_sampled(nat):
    """Prefill single linear at full size (M=2048, K=4096, N=11008), plain and
    with the fused ReLU; sampled rows x channels recomputed by the oracle."""
    c = synth.prefill_case()
    wpd, swd = nat.w4_quantize_pack(dev(c.w))
    rng = synth.rng_for(10, 10)
    rows = np.unique(np.concatenate([[0, 2047], rng.integers(0, 2048, size=6)]))
    cols = np.unique(np.concatenate([[0, 11007], rng.integers(0, 11008, size=60)]))
    for relu in (False, True):
        _sampled_check(nat, c.x, c.w, wpd, swd, rows, cols, relu=relu)


@pytest.mark.parametrize("shape", [0, 1])
def test_llama70_shapes_sampled(nat, shape):
    """70B-shaped linears at full size for M in {1, 16, 128, 4096}."""
    c0 = synth.llama70_case(shape, 1, with_x=False)
    k, n = synth.LLAMA70_SHAPES[shape]
    wpd, swd = nat.w4_quantize_pack(dev(c0.w))
    rng = synth.rng_for(11, shape)
    cols = np.unique(np.concatenate([[0, n - 1], rng.integers(0, n, size=40)]))
    wp_ref, sw_ref = oracle.w4_quantize_pack(c0.w[:, cols])
    assert np.array_equal(host(wpd)[cols], wp_ref)
    assert np.array_equal(host(swd)[cols], sw_ref)
    for m in synth.LLAMA70_MS:
        c = synth.llama70_case(shape, m)
        rows = np.unique(np.concatenate([[0, m - 1], rng.integers(0, m, size=4)]))
        _sampled_check(nat, c.x, None, wpd, swd, rows, cols)


@pytest.mark.parametrize("path", PATHS)
def test_linear_q_full_code_range(nat, path):
    """Every INT4 code, -8 included (the packed format allows it even though
    abs-max quantization never produces it), against every INT8 value."""
    rng = synth.rng_for(12, 0)
    m, k, n = 40, 768, 136
    q = rng.integers(-8, 8, size=(n, k)).astype(np.int8)
    q[:, :16] = -8
    xq = rng.integers(-127, 128, size=(m, k)).astype(np.int8)
    xq[:, :16] = -127
    sx = (rng.random(m) + 0.5).astype(np.float32)
    sw = (rng.random(n) + 0.5).astype(np.float32)
    wp = oracle.w4_pack(q)
    acc = nat.w4a8_linear_q(dev(xq), dev(sx), k, dev(wp), dev(sw), out="s32", path=path)
    assert np.array_equal(host(acc), oracle.gemm_s32(xq, k, wp))
    y = nat.w4a8_linear_q(dev(xq), dev(sx), k, dev(wp), dev(sw), path=path)
    assert_f32_close(host(y), oracle.linear_q(xq, sx, wp, sw, k))


def test_tc_large_k_uses_sign_extension(nat):
    """K above the limit of the tensor-core kernel's 16*q byte trick
    (each term 16 q * xq is at most 128 * 127 in size, so 128 * 127 * K must
    stay below 2^31) still gives exact results."""
    m, k, n = 20, 140000, 16
    x, w, _ = _case(m, k, n, seed=900)
    wp, sw = oracle.w4_quantize_pack(w)
    acc = nat.w4a8_linear(dev(x), dev(wp), dev(sw), out="s32", path="tc")
    assert np.array_equal(host(acc), oracle.linear(x, wp, sw, k, out="s32"))


@pytest.mark.parametrize("m,k,n,pad", [(1, 4096, 64, 0), (5, 1001, 40, 3), (8, 2048, 33, 0)])
def test_decode_linear_matches_quantize_then_linear_q(nat, m, k, n, pad):
    """w4a8_linear on the decode path must agree bit for bit with quantizing
    first (a8_quantize_rows) and multiplying after (w4a8_linear_q), and with
    the oracle. `pad` widens the row stride so float4 loads are ruled out."""
    x, w, b = _case(m, k, n, seed=1000 + m)
    if m > 2:
        x[2] = 0.0
    xbuf = np.zeros((m, k + pad), np.float32)
    xbuf[:, :k] = x
    xd = dev(xbuf)[:, :k]
    wp, sw = oracle.w4_quantize_pack(w)
    wpd, swd, bd = dev(wp), dev(sw), dev(b)
    y1 = nat.w4a8_linear(xd, wpd, swd, bias=bd, path="decode")
    xq, sx = nat.a8_quantize_rows(xd)
    y2 = nat.w4a8_linear_q(xq, sx, k, wpd, swd, bias=bd, path="decode")
    a, c = host(y1), host(y2)
    assert np.array_equal(a.view(np.uint32), c.view(np.uint32))
    assert_f32_close(a, oracle.linear(x, wp, sw, k, bias=b), b)


# ------------------------------------- decode with fused quantization ---

@pytest.mark.parametrize("m", [1, 2, 3, 4])
@pytest.mark.parametrize("k,pad", [(1, 0), (7, 1), (129, 0), (4100, 0), (4100, 3)])
def test_fused_decode_bit_exact(nat, m, k, pad):
    """Few-row decode quantizes X inside the product kernel: the INT32
    accumulators must be the oracle's bit for bit (a zero row included), the
    float outputs within the layer tolerance, with and without the
    static-weights promise. `pad` rules out float4 loads of X."""
    n = 40
    x, w, b = _case(m, k, n, seed=1100 + 7 * m + k)
    if m > 1:
        x[1] = 0.0
    xbuf = np.zeros((m, k + pad), np.float32)
    xbuf[:, :k] = x
    xd = dev(xbuf)[:, :k]
    wp, sw = oracle.w4_quantize_pack(w)
    wpd, swd, bd = dev(wp), dev(sw), dev(b)
    acc_ref = oracle.linear(x, wp, sw, k, out="s32")
    for static in (False, True):
        acc = nat.w4a8_linear(xd, wpd, swd, out="s32", path="decode", static_weights=static)
        assert nat.last_path() == "decode"
        assert np.array_equal(host(acc), acc_ref)
        y = nat.w4a8_linear(xd, wpd, swd, bias=bd, relu=True, path="decode", static_weights=static)
        assert_f32_close(host(y), oracle.linear(x, wp, sw, k, bias=b, relu=True), b)
        yb = nat.w4a8_linear(xd, wpd, swd, bias=bd, out="bf16", path="decode", static_weights=static)
        assert_bf16_within_ulp(host(yb.view(torch.int16)),
                               oracle.linear(x, wp, sw, k, bias=b, out="bf16"))


@pytest.mark.parametrize("m,k", [(1, 8192), (1, 8193), (2, 4096), (2, 4097), (4, 2048), (4, 2049),
                                 (1, 65536), (1, 65537), (2, 32768), (2, 32769), (4, 16384), (4, 16385),
                                 (8, 8192), (8, 8193)])
@pytest.mark.parametrize("path", ["decode", "ring"])
def test_decode_at_kernel_boundaries(nat, m, k, path):
    """Both sides of every K at which the few-row decode changes kernels: the
    activation quantization still fits the ring kernel's registers; one ring
    stage and the INT8 rows still fit a block's shared memory. The result
    must not depend on the side, with or without the static-weights
    promise."""
    n = 24
    x, w, _ = _case(m, k, n, seed=1200 + m)
    wp, sw = oracle.w4_quantize_pack(w)
    ref = oracle.linear(x, wp, sw, k, out="s32")
    for static in (False, True):
        try:
            acc = nat.w4a8_linear(dev(x), dev(wp), dev(sw), out="s32", path=path, static_weights=static)
        except nat.W4A8Error as e:
            # forced onto the ring past its shared-memory budget (the odd-K side
            # of the boundaries that fall there): refused, nothing enqueued
            assert path == "ring" and k % 2 == 1 and e.status == nat.ERR_UNSUPPORTED
            continue
        assert np.array_equal(host(acc), ref)


@pytest.mark.parametrize("m", [1, 4, 16, 300])
def test_static_weights_promise_gives_same_bits(nat, m):
    """W4A8_STATIC_WEIGHTS only lets kernels read the weights earlier: the
    outputs of w4a8_linear and w4a8_linear_q are the same bits either way."""
    k, n = 1024, 520
    x, w, b = _case(m, k, n, seed=1300 + m)
    wpd, swd = nat.w4_quantize_pack(dev(w))
    xd, bd = dev(x), dev(b)
    torch.cuda.synchronize()                 # the weights are settled from here on
    y0 = host(nat.w4a8_linear(xd, wpd, swd, bias=bd))
    y1 = host(nat.w4a8_linear(xd, wpd, swd, bias=bd, static_weights=True))
    assert np.array_equal(y0.view(np.uint32), y1.view(np.uint32))
    xq, sx = nat.a8_quantize_rows(xd)
    q0 = host(nat.w4a8_linear_q(xq, sx, k, wpd, swd, bias=bd))
    q1 = host(nat.w4a8_linear_q(xq, sx, k, wpd, swd, bias=bd, static_weights=True))
    assert np.array_equal(q0.view(np.uint32), q1.view(np.uint32))
    assert np.array_equal(y0.view(np.uint32), q0.view(np.uint32))


@pytest.mark.parametrize("m", [2, 3, 4])
def test_fused_two_pass_decode_sampled(nat, m):
    """Few rows against a long weight stream (K = 8192, N = 28672): the decode
    kernel quantizes X in two passes of its own; sampled channels against the
    oracle, plus bit-equality with quantizing first (a8_quantize_rows) and
    multiplying after (w4a8_linear_q)."""
    c0 = synth.llama70_case(0, 1, with_x=False)
    k, n = synth.LLAMA70_SHAPES[0]
    wpd, swd = nat.w4_quantize_pack(dev(c0.w))
    x, _ = synth.linear_activations(m, k, seed=1400 + m, outlier_count=8, outlier_factor=50.0)
    rng = synth.rng_for(14, m)
    cols = np.unique(np.concatenate([[0, n - 1], rng.integers(0, n, size=40)]))
    y = _sampled_check(nat, x, None, wpd, swd, np.arange(m), cols, path="decode")
    assert nat.last_launch_count() == 1
    xq, sx = nat.a8_quantize_rows(dev(x))
    yq = host(nat.w4a8_linear_q(xq, sx, k, wpd, swd, path="decode"))
    assert np.array_equal(np.asarray(y).view(np.uint32), yq.view(np.uint32))


def test_bounded_wait_gives_up_and_reports(nat):
    """Failure detection without a GPU fault: a wait that nothing satisfies
    gives up after its limit, the device status word reads W4A8_ERR_TIMEOUT,
    and the context keeps working."""
    nat.get_device_status(clear=True)
    nat.selftest_timeout(1_000_000)
    assert nat.get_device_status(clear=True) == nat.ERR_TIMEOUT
    assert nat.get_device_status() == nat.OK
    m, k, n = 3, 64, 16
    x, w, _ = _case(m, k, n, seed=1500)
    wp, sw = oracle.w4_quantize_pack(w)
    acc = nat.w4a8_linear(dev(x), dev(wp), dev(sw), out="s32")
    assert np.array_equal(host(acc), oracle.linear(x, wp, sw, k, out="s32"))


# ------------------------------------------------------ grouped decode ---

def _grouped_case(specs, seed):
    probs, refs = [], []
    for i, (m, k, n, with_bias) in enumerate(specs):
        x, w, b = _case(m, k, n, seed=seed + i)
        if m > 1:
            x[m - 1] = 0.0                     # an all-zero row
        wp, sw = oracle.w4_quantize_pack(w)
        probs.append((x, wp, sw, b if with_bias else None))
    return probs


@pytest.mark.parametrize("out", ["f32", "bf16", "s32"])
def test_grouped_decode_matches_single_calls(nat, out):
    """Heterogeneous problems (K from 1 to 6912, odd K, N tails, M 1..4, some
    with a bias) in one grouped call give the same bits as one w4a8_linear per
    problem, and the INT32 accumulators equal the oracle's."""
    specs = [(1, 4096, 4096, True), (4, 1152, 1024, False), (2, 7, 40, True), (3, 6912, 1152, True),
             (1, 1, 17, False), (4, 4100, 300, True), (1, 1152, 256, False), (2, 999, 96, False)]
    probs = _grouped_case(specs, seed=1600)
    relu = out != "s32"
    dp = [(dev(x), dev(wp), dev(sw), None if (b is None or out == "s32") else dev(b)) for x, wp, sw, b in probs]
    ys = nat.w4a8_linear_grouped(dp, relu=relu, out=out)
    assert nat.last_launch_count() == 1
    for (x, wp, sw, b), (xd, wpd, swd, bd), y in zip(probs, dp, ys):
        y1 = nat.w4a8_linear(xd, wpd, swd, bias=bd, relu=relu, out=out)
        a = host(y.view(torch.int32) if out != "bf16" else y.view(torch.int16))
        b1 = host(y1.view(torch.int32) if out != "bf16" else y1.view(torch.int16))
        assert np.array_equal(a, b1)
        k = x.shape[1]
        if out == "s32":
            assert np.array_equal(host(y), oracle.linear(x, wp, sw, k, out="s32"))
        elif out == "bf16":
            assert_bf16_within_ulp(a, oracle.linear(x, wp, sw, k, bias=b, relu=relu, out="bf16"))
        else:
            assert_f32_close(host(y), oracle.linear(x, wp, sw, k, bias=b, relu=relu), b)


def test_grouped_decode_many_problems_and_static_weights(nat):
    """More problems than one launch holds (70 of them), M = 0 problems
    skipped, and the static-weights promise: same bits as single calls."""
    specs = [((i % 4) + 1, 64 * (1 + i % 9), 16 * (1 + i % 5) + (i % 3), i % 2 == 0) for i in range(70)]
    probs = _grouped_case(specs, seed=1700)
    dp = [(dev(x), dev(wp), dev(sw), None if b is None else dev(b)) for x, wp, sw, b in probs]
    empty = (torch.empty((0, 64), device="cuda"), dp[0][1], dp[0][2], None)
    torch.cuda.synchronize()
    ys = nat.w4a8_linear_grouped(dp[:35] + [empty] + dp[35:], static_weights=True)
    assert nat.last_launch_count() == 2
    ys = ys[:35] + ys[36:]
    for (xd, wpd, swd, bd), y in zip(dp, ys):
        y1 = nat.w4a8_linear(xd, wpd, swd, bias=bd)
        assert np.array_equal(host(y).view(np.uint32), host(y1).view(np.uint32))


@pytest.mark.parametrize("path", ["tc", "decode", "generic", "split", "ring", "regs"])
def test_extreme_scale_products(nat, path):
    """Rows and weight columns whose scales are finite but whose product
    sx * sw leaves the normal float32 range: row 0 has abs-max ~5e-32
    (sx ~2.5e33) and meets a weight column of abs-max ~3e-9 (sw ~2.2e9), so
    sx * sw overflows to inf and y = acc / inf is a signed zero; row 1 has
    abs-max ~2.4e34 (sx ~5e-33) and meets a column of abs-max ~3.4e20
    (sw ~2e-20), so sx * sw underflows to 0 and y = acc / 0 is infinite; row
    1 against the ordinary columns gives sx * sw ~2^-100, below the range of
    the reciprocal form. Every path must give the oracle's IEEE results there,
    and the 1e-6 bar elsewhere."""
    m, k, n = (8 if path in ("split", "ring") else 40), 512, 48
    x, w, _ = _case(m, k, n, seed=990)
    x[0] *= 1e-33
    x[1] *= 1e33
    w[:, 0] *= 1e-9 / 0.02
    w[:, 1] *= 1e20 / 0.02
    wp, sw = oracle.w4_quantize_pack(w)
    ref = oracle.linear(x, wp, sw, k)
    got = host(nat.w4a8_linear(dev(x), dev(wp), dev(sw), path=path))
    special = ~np.isfinite(ref) | (ref == 0)
    assert special[0, 0] and special[1, 1]
    signed = special & ~np.isnan(ref)          # a NaN's sign bit is not defined by IEEE division
    assert np.array_equal(np.signbit(got[signed]), np.signbit(ref[signed]))
    assert np.array_equal(got[special], ref[special], equal_nan=True)
    assert_f32_close(np.where(special, 1.0, got), np.where(special, 1.0, ref))
