"""Pins for the CPU oracle: what the pages and the mathematics fix, checked
against something other than the oracle itself (hand-worked fixtures, closed
forms, invariants, brute force, library routines, error bounds).

Method: Keras guide "INT4 quantization in Keras", section "How it works",
steps 1-6; the minimal model of section "Quantize a minimal functional model".
"""
import itertools
import math

import numpy as np
import pytest
import torch

import oracle
from tests.conftest import read_golden
from w4a8_quantized_gemm_channel_b200 import synth


def _ints(vals):
    return [int(v) for v in vals]


# ---------------------------------------------------------------- packing ---

def test_pack_matches_hand_worked_bytes():
    """The nibble order and two's-complement encoding, worked by hand for
    every code value in both nibble positions, plus an odd K."""
    rows = read_golden("pack_codes.txt")
    assert len(rows) % 2 == 0 and rows
    for (k1, codes), (k2, hexbytes) in zip(rows[::2], rows[1::2]):
        assert k1 == "codes" and k2 == "bytes"
        q = np.array([_ints(codes)], np.int8)
        wp = oracle.w4_pack(q)
        want = bytes(int(h, 16) for h in hexbytes)
        assert wp.shape[1] == oracle.packed_ld(q.shape[1])
        assert bytes(wp[0, :len(want)]) == want
        assert not wp[0, len(want):].any(), "pad bytes must be zero"
        # and unpacking gives the codes back
        assert np.array_equal(oracle.w4_unpack(wp, q.shape[1]), q)


def test_pack_unpack_round_trip_exhaustive():
    """unpack(pack(q)) == q for every pair of codes in [-8, 7], and
    pack(unpack(b)) == b for every byte value."""
    pairs = np.array(list(itertools.product(range(-8, 8), repeat=2)), np.int8)  # 256 x 2
    wp = oracle.w4_pack(pairs)
    assert np.array_equal(oracle.w4_unpack(wp, 2), pairs)
    # every byte value occurs exactly once among the packed pairs
    assert sorted(wp[:, 0].tolist()) == list(range(256))
    allbytes = np.zeros((256, 16), np.uint8)
    allbytes[:, 0] = np.arange(256)
    q = oracle.w4_unpack(allbytes, 2)
    assert q.min() == -8 and q.max() == 7
    assert np.array_equal(oracle.w4_pack(q)[:, 0], np.arange(256))


def test_packed_size_is_params_times_bits_over_8():
    """Size = parameters x 4 bits / 8 (the concept page's storage formula),
    before the row padding to 16 bytes."""
    for k in (1, 2, 3, 31, 32, 33, 4096, 6912):
        assert oracle.packed_ld(k) >= math.ceil(k * 4 / 8)
        assert oracle.packed_ld(k) - math.ceil(k * 4 / 8) < 16
        assert oracle.packed_ld(k) % 16 == 0


# --------------------------------------------------------------- rounding ---

def test_weight_ties_round_half_even():
    g = dict(read_golden("round_half_even.txt"))
    w = np.array([float(v) for v in g["weight_column"]], np.float32)[:, None]
    q, sw = oracle.w4_quantize(w)
    assert sw[0] == np.float32(1.0)
    assert q[0].tolist() == _ints(g["weight_codes"])


def test_activation_ties_round_half_even():
    g = dict(read_golden("round_half_even.txt"))
    x = np.array([[float(v) for v in g["act_row"]]], np.float32)
    xq, sx = oracle.a8_quantize_rows(x)
    assert sx[0] == np.float32(1.0)
    assert xq[0].tolist() == _ints(g["act_codes"])


# ------------------------------------------------------ weight quantization ---

def _random_w(k=384, n=96, seed=11):
    return synth.linear_weights(k, n, 0.02, seed)


def test_weight_codes_in_range_and_extremes_hit_7():
    """Codes stay in [-8, 7]; with abs-max scaling to 7 they never reach -8,
    and the element attaining a column's abs-max maps to exactly +-7."""
    w = _random_w()
    q, sw = oracle.w4_quantize(w)
    assert q.min() >= -7 and q.max() <= 7
    for n in range(w.shape[1]):
        kmax = int(np.argmax(np.abs(w[:, n])))
        assert q[n, kmax] == (7 if w[kmax, n] > 0 else -7)
    # the scale is 7 / abs-max (float32 division)
    amax = np.abs(w).max(axis=0)
    assert np.array_equal(sw, (np.float32(7.0) / amax).astype(np.float32))


def test_weight_scale_invariance_by_powers_of_two():
    """Scaling a column by 2^j leaves its codes unchanged and divides its
    scale by exactly 2^j (both products are exact in binary floating point)."""
    w = _random_w(k=200, n=8, seed=12)
    q0, sw0 = oracle.w4_quantize(w)
    for j in (-3, 1, 5):
        wj = (w * np.float32(2.0 ** j)).astype(np.float32)
        qj, swj = oracle.w4_quantize(wj)
        assert np.array_equal(qj, q0)
        assert np.array_equal(swj * np.float32(2.0 ** j), sw0)


def test_weight_sign_symmetry():
    """Round-half-even is odd-symmetric, so Q(-W) = -Q(W) with the same scale."""
    w = _random_w(k=256, n=16, seed=13)
    q0, sw0 = oracle.w4_quantize(w)
    q1, sw1 = oracle.w4_quantize(-w)
    assert np.array_equal(sw0, sw1)
    assert np.array_equal(q1, -q0)


def test_zero_column_and_zero_row():
    w = _random_w(k=64, n=4, seed=14)
    w[:, 2] = 0.0
    q, sw = oracle.w4_quantize(w)
    assert sw[2] == np.float32(1.0) and not q[2].any()
    x = synth.normal((3, 64), 1.0, synth.rng_for(14, 9))
    x[1] = 0.0
    xq, sx = oracle.a8_quantize_rows(x)
    assert sx[1] == np.float32(1.0) and not xq[1].any()


def test_weight_error_bound():
    """|w - q/sw| <= 0.5/sw for every element: no value is clipped (the
    abs-max maps to 7 < 8), so rounding is the only error."""
    w = _random_w(k=512, n=64, seed=15).astype(np.float64)
    q, sw = oracle.w4_quantize(w.astype(np.float32))
    sw64 = sw.astype(np.float64)
    err = np.abs(w.T - q.astype(np.float64) / sw64[:, None])
    bound = 0.5 / sw64[:, None] * (1 + 1e-6)
    assert (err <= bound).all()


# -------------------------------------------------- activation quantization ---

def test_activation_codes_range_extremes_and_error_bound():
    x, _ = synth.linear_activations(16, 1000, seed=16, outlier_count=5, outlier_factor=20.0)
    xq, sx = oracle.a8_quantize_rows(x)
    assert xq.min() >= -127 and xq.max() <= 127
    for m in range(x.shape[0]):
        k = int(np.argmax(np.abs(x[m])))
        assert xq[m, k] == (127 if x[m, k] > 0 else -127)
    assert np.array_equal(sx, (np.float32(127.0) / np.abs(x).max(axis=1)).astype(np.float32))
    err = np.abs(x.astype(np.float64) - xq.astype(np.float64) / sx.astype(np.float64)[:, None])
    assert (err <= 0.5 / sx.astype(np.float64)[:, None] * (1 + 1e-6)).all()


def test_activation_pad_bytes_are_zero():
    x = synth.normal((5, 37), 1.0, synth.rng_for(17, 1))
    xq, _ = oracle.a8_quantize_rows(x, ldq=48)
    assert not xq[:, 37:].any()


# ---------------------------------------------------------------- the GEMM ---

def test_gemm_brute_force_exhaustive_tiny():
    """Every weight code vector in [-8, 7]^K for K <= 3 against fixed
    activation rows (extremes included), checked with a pure-Python loop."""
    for k in (1, 2, 3):
        q = np.array(list(itertools.product(range(-8, 8), repeat=k)), np.int8)  # N x K
        xq = np.array([[127] * k, [-127] * k, list(range(1, k + 1)),
                       [(-1) ** i * (30 + 11 * i) for i in range(k)]], np.int8)
        acc = oracle.gemm_s32(xq, k, oracle.w4_pack(q))
        for m in range(xq.shape[0]):
            for n in range(q.shape[0]):
                s = 0
                for kk in range(k):
                    s += int(xq[m, kk]) * int(q[n, kk])
                assert acc[m, n] == s


def test_gemm_brute_force_small_random():
    rng = synth.rng_for(18, 0)
    for (m, k, n) in ((1, 1, 1), (3, 7, 5), (4, 8, 4), (2, 33, 3)):
        q = rng.integers(-8, 8, size=(n, k)).astype(np.int8)
        xq = rng.integers(-127, 128, size=(m, k)).astype(np.int8)
        acc = oracle.gemm_s32(xq, k, oracle.w4_pack(q))
        want = [[sum(int(xq[i, t]) * int(q[j, t]) for t in range(k)) for j in range(n)]
                for i in range(m)]
        assert acc.tolist() == want


def test_gemm_matches_float64_matmul_medium():
    """Integer products summed in float64 are exact while |acc| < 2^53."""
    rng = synth.rng_for(19, 0)
    m, k, n = 24, 777, 40
    q = rng.integers(-8, 8, size=(n, k)).astype(np.int8)
    xq = rng.integers(-127, 128, size=(m, k)).astype(np.int8)
    acc = oracle.gemm_s32(xq, k, oracle.w4_pack(q))
    ref = xq.astype(np.float64) @ q.astype(np.float64).T
    assert np.array_equal(acc.astype(np.float64), ref)


def test_gemm_int32_overflow_is_reported():
    k = 2_200_000  # 127 * 8 * k > 2^31
    xq = np.full((1, k), -127, np.int8)
    q = np.full((1, k), -8, np.int8)
    with pytest.raises(oracle.OracleError):
        oracle.gemm_s32(xq, k, oracle.w4_pack(q))


# --------------------------------------------------------- dequantization ---

def test_dequant_direction_exact_powers_of_two():
    """With abs-maxes 3.5 and 63.5 both scales are exactly 2, every value is a
    half-integer and exactly representable, so y must equal X @ W exactly:
    y = acc / (sx * sw) = acc / 4. Dividing by sx/sw or multiplying by
    sx*sw instead would miss by a factor of 4 or 16."""
    rng = synth.rng_for(20, 0)
    m, k, n = 6, 50, 9
    wq = rng.integers(-7, 8, size=(k, n)).astype(np.float32)
    wq[0, :] = 7
    xq = rng.integers(-127, 128, size=(m, k)).astype(np.float32)
    xq[:, 0] = 127
    w = wq / 2   # abs-max 3.5 -> sw = 2
    x = xq / 2   # abs-max 63.5 -> sx = 2
    wp, sw = oracle.w4_quantize_pack(w)
    assert (sw == 2.0).all()
    y = oracle.linear(x, wp, sw, k)
    exact = x.astype(np.float64) @ w.astype(np.float64)
    assert np.array_equal(y.astype(np.float64), exact)


def test_dequant_bias_and_relu():
    acc = np.array([[-10, 0, 10, 3]], np.int32)
    sx = np.array([2.0], np.float32)
    sw = np.array([1.0, 1.0, 0.5, 4.0], np.float32)
    b = np.array([4.0, -1.0, 0.5, 0.0], np.float32)
    y = oracle.dequant(acc, sx, sw, b, relu=False)
    assert y.tolist() == [[-1.0, -1.0, 10.5, 0.375]]
    y = oracle.dequant(acc, sx, sw, b, relu=True)
    assert y.tolist() == [[0.0, 0.0, 10.5, 0.375]]
    assert not np.signbit(y).any()


def test_end_to_end_error_bound():
    """|y_q - y_exact| <= sum_k (|x_k| e_w + |w_k| e_x + e_w e_x) + float32
    slack, with e_w = 0.5/sw and e_x = 0.5/sx and y_exact = X @ W in float64.
    A swapped scale convention or a dropped factor breaks this bound."""
    x, _ = synth.linear_activations(8, 640, seed=21, outlier_count=3, outlier_factor=20.0)
    w = synth.linear_weights(640, 48, 0.02, seed=21)
    wp, sw = oracle.w4_quantize_pack(w)
    xq, sx = oracle.a8_quantize_rows(x)
    y = oracle.linear(x, wp, sw, 640)
    x64, w64 = x.astype(np.float64), w.astype(np.float64)
    exact = x64 @ w64
    ew = 0.5 / sw.astype(np.float64)            # [N]
    ex = 0.5 / sx.astype(np.float64)            # [M]
    bound = (np.abs(x64).sum(1)[:, None] * ew[None, :]
             + ex[:, None] * np.abs(w64).sum(0)[None, :]
             + 640 * ex[:, None] * ew[None, :])
    slack = 1e-5 * (np.abs(x64) @ np.abs(w64)) + 1e-6
    assert (np.abs(y - exact) <= bound + slack).all()
    # and the error is not trivially zero: quantization happened
    assert np.abs(y - exact).max() > 0


def test_bf16_rounding_matches_torch():
    """float32 -> bf16 round-to-nearest-even agrees with torch's conversion."""
    rng = synth.rng_for(22, 0)
    y = np.concatenate([rng.standard_normal(4096).astype(np.float32) * 100,
                        np.array([0.0, -0.0, 1.0, 1.00390625, 1.01171875, -3.0e38, 1e-40],
                                 np.float32)])
    want = torch.from_numpy(y).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(oracle.to_bf16_bits(y), want)


# -------------------------------------------------------- minimal model ---

def _fp_mlp(d: synth.MinimalMLP) -> np.ndarray:
    x = d.x.astype(np.float64)
    h = np.maximum(x @ d.w1.astype(np.float64) + d.b1, 0.0)
    return h @ d.w2.astype(np.float64) + d.b2


def test_minimal_model_mse_order_of_magnitude():
    """The page's minimal model: quantized vs full-precision MSE is small and
    of the order the page prints (its data are unseeded: order only)."""
    page = float(dict(read_golden("minimal_mlp_mse.txt"))["page_mse"][0])
    d = synth.minimal_mlp(seed=0)
    yq = oracle.mlp(d.x, d.w1, d.b1, d.w2, d.b2)
    mse = float(np.mean((_fp_mlp(d) - yq.astype(np.float64)) ** 2))
    assert 0.0 < mse <= 1e-2
    assert page / 100 <= mse <= page * 100, (mse, page)


def test_minimal_model_is_deterministic():
    """Re-running the quantized model gives bit-identical outputs (the page's
    save/reload MSE is identical for the same reason: the quantized state is
    just packed bytes and scales)."""
    d = synth.minimal_mlp(seed=0)
    a = oracle.mlp(d.x, d.w1, d.b1, d.w2, d.b2)
    b = oracle.mlp(d.x, d.w1, d.b1, d.w2, d.b2)
    assert np.array_equal(a.view(np.uint32), b.view(np.uint32))


# ------------------------------------------------------------------ W8A8 ---
# The INT8 path the page presents INT4 as an extension of (section "How it
# works", closing paragraph): 8-bit codes, scale 127 / abs-max, no packing.

def test_w8_codes_hand_worked():
    """Abs-max 1 gives sw = 127; 0.5 * 127 = 63.5 is a tie and rounds to the
    even 64 (-63.5 to -64), 0.25 * 127 = 31.75 rounds to 32, and the abs-max
    element maps to 127. Pad bytes past K are 0."""
    w = np.array([[1.0], [-0.5], [0.25], [0.5], [-1.0]], np.float32)
    q8, sw = oracle.w8_quantize(w, ldw8=16)
    assert sw.tolist() == [127.0]
    assert q8[0, :5].tolist() == [127, -64, 32, 64, -127]
    assert not q8[0, 5:].any()


def test_w8_codes_range_extremes_and_scale():
    """Codes stay in [-127, 127]; the element attaining a column's abs-max maps
    to exactly +-127; the scale is 127 / abs-max in float32."""
    w = _random_w(k=300, n=40, seed=31)
    q8, sw = oracle.w8_quantize(w)
    assert q8.min() >= -127 and q8.max() <= 127
    for n in range(w.shape[1]):
        kmax = int(np.argmax(np.abs(w[:, n])))
        assert q8[n, kmax] == (127 if w[kmax, n] > 0 else -127)
    amax = np.abs(w).max(axis=0)
    assert np.array_equal(sw, (np.float32(127.0) / amax).astype(np.float32))


def test_w8_invariances_and_zero_column():
    """Powers of two leave the codes unchanged and divide the scale exactly;
    negating W negates the codes; an all-zero column has scale 1, codes 0."""
    w = _random_w(k=200, n=8, seed=32)
    w[:, 5] = 0.0
    q0, sw0 = oracle.w8_quantize(w)
    assert sw0[5] == np.float32(1.0) and not q0[5].any()
    for j in (-4, 3):
        qj, swj = oracle.w8_quantize((w * np.float32(2.0 ** j)).astype(np.float32))
        assert np.array_equal(qj, q0)
        nz = np.arange(w.shape[1]) != 5  # the zero column keeps scale 1
        assert np.array_equal((swj * np.float32(2.0 ** j))[nz], sw0[nz]) and swj[5] == 1.0
    q1, sw1 = oracle.w8_quantize(-w)
    assert np.array_equal(sw1, sw0) and np.array_equal(q1, -q0)


def test_w8_weight_error_bound():
    """|w - q/sw| <= 0.5/sw everywhere: the abs-max maps to 127, nothing clips."""
    w = _random_w(k=512, n=64, seed=33).astype(np.float64)
    q8, sw = oracle.w8_quantize(w.astype(np.float32))
    err = np.abs(w.T - q8[:, :512].astype(np.float64) / sw.astype(np.float64)[:, None])
    assert (err <= 0.5 / sw.astype(np.float64)[:, None] * (1 + 1e-6)).all()


def test_gemm8_matches_float64_matmul():
    """Integer products summed in float64 are exact while |acc| < 2^53; the
    codes span the full INT8 range on both sides, pad bytes are ignored."""
    rng = synth.rng_for(34, 0)
    for (m, k, n) in ((1, 1, 1), (3, 7, 5), (24, 777, 40)):
        q8 = np.zeros((n, (k + 15) // 16 * 16), np.int8)
        q8[:, :k] = rng.integers(-127, 128, size=(n, k))
        q8[:, k:] = 99  # pad bytes: must not be read
        xq = rng.integers(-127, 128, size=(m, k)).astype(np.int8)
        acc = oracle.gemm8_s32(xq, k, q8)
        ref = xq.astype(np.float64) @ q8[:, :k].astype(np.float64).T
        assert np.array_equal(acc.astype(np.float64), ref)


def test_gemm8_int32_overflow_is_reported():
    k = 133_200  # 127 * 127 * k > 2^31 - 1
    xq = np.full((1, k), 127, np.int8)
    q8 = np.full((1, k), 127, np.int8)
    with pytest.raises(oracle.OracleError):
        oracle.gemm8_s32(xq, k, q8)
    k = 133_144  # the largest K whose worst case fits
    assert oracle.gemm8_s32(xq[:, :k], k, q8[:, :k])[0, 0] == 127 * 127 * k


def test_linear8_exact_when_codes_are_exact():
    """Abs-maxes 63.5 (X) and 63.5 (W) give sx = sw = 2; every value is a
    half-integer, so y = acc / 4 equals X @ W exactly (a swapped or dropped
    scale misses by a factor of 4 or 16)."""
    rng = synth.rng_for(35, 0)
    m, k, n = 5, 60, 7
    wq = rng.integers(-127, 128, size=(k, n)).astype(np.float32)
    wq[0, :] = 127
    xq = rng.integers(-127, 128, size=(m, k)).astype(np.float32)
    xq[:, 0] = -127
    w, x = wq / 2, xq / 2
    q8, sw = oracle.w8_quantize(w)
    assert (sw == 2.0).all()
    y = oracle.linear8(x, q8, sw, k)
    assert np.array_equal(y.astype(np.float64), x.astype(np.float64) @ w.astype(np.float64))


def test_linear8_error_bound_and_tighter_than_int4():
    """The same error bound as the INT4 layer with e_w = 0.5/sw, sw = 127 /
    abs-max; on the same data the INT8 weights' error is well below INT4's."""
    x, _ = synth.linear_activations(8, 640, seed=36, outlier_count=3, outlier_factor=20.0)
    w = synth.linear_weights(640, 48, 0.02, seed=36)
    q8, sw = oracle.w8_quantize(w)
    xq, sx = oracle.a8_quantize_rows(x)
    y8 = oracle.linear8(x, q8, sw, 640)
    x64, w64 = x.astype(np.float64), w.astype(np.float64)
    exact = x64 @ w64
    ew = 0.5 / sw.astype(np.float64)
    ex = 0.5 / sx.astype(np.float64)
    bound = (np.abs(x64).sum(1)[:, None] * ew[None, :] + ex[:, None] * np.abs(w64).sum(0)[None, :]
             + 640 * ex[:, None] * ew[None, :])
    slack = 1e-5 * (np.abs(x64) @ np.abs(w64)) + 1e-6
    assert (np.abs(y8 - exact) <= bound + slack).all()
    wp, sw4 = oracle.w4_quantize_pack(w)
    y4 = oracle.linear(x, wp, sw4, 640)
    assert np.abs(y8 - exact).mean() < 0.5 * np.abs(y4 - exact).mean()


# ------------------------------------------------ asymmetric INT4 (zero point) ---
# "INT4" concept page, section 4.1 (asymmetric uniform quantization) and the
# "4-bit Integer Quantization for LLMs" page, section "Weight quantization".

def _unpack_unsigned(wp, k):
    """Nibbles of each packed row as unsigned codes, written independently of the oracle."""
    lo = (wp & 0x0F).astype(np.int64)
    hi = (wp >> 4).astype(np.int64)
    codes = np.empty((wp.shape[0], 2 * wp.shape[1]), np.int64)
    codes[:, 0::2], codes[:, 1::2] = lo, hi
    return codes[:, :k]


def test_w4z_hand_worked_codes():
    """Column [-1, 0, 2, 0.5]: range 3 -> sa = 15/3 = 5, zp = -rne(-5) = 5;
    codes -5+5 = 0, 0+5 = 5, 10+5 = 15, rne(2.5) = 2 (tie to even) + 5 = 7;
    bytes 0 | 5 << 4 = 80 and 15 | 7 << 4 = 127, pad 0."""
    w = np.array([[-1.0], [0.0], [2.0], [0.5]], np.float32)
    wp, sa, zp = oracle.w4z_quantize_pack(w)
    assert sa.tolist() == [5.0] and zp.tolist() == [5]
    assert wp[0, :2].tolist() == [80, 127] and not wp[0, 2:].any()


def test_w4z_clamp_binds_on_a_tie_at_the_top():
    """Column [-0.5, 0.5, 0]: sa = 15, zp = -rne(-7.5) = 8 (tie to even);
    0.5 * 15 = 7.5 also rounds to 8, and 8 + 8 = 16 must clamp to 15 (not wrap
    to 0); 0 maps to 8. Bytes 0 | 15 << 4 = 240 and 8."""
    w = np.array([[-0.5], [0.5], [0.0]], np.float32)
    wp, sa, zp = oracle.w4z_quantize_pack(w)
    assert sa.tolist() == [15.0] and zp.tolist() == [8]
    assert wp[0, :2].tolist() == [240, 8]


def test_w4z_range_ends_and_dequant_error():
    """Each column's minimum maps to code 0 and its maximum to 15; every code is
    in [0, 15]; the dequantized weight (q - zp) / sa is within 0.5 / sa of w
    except where the clamp took a tie at the top from 16 to 15 (then 1 / sa)."""
    w = _random_w(k=300, n=40, seed=41)
    wp, sa, zp = oracle.w4z_quantize_pack(w)
    q = _unpack_unsigned(wp, 300)
    assert q.min() >= 0 and q.max() <= 15
    for n in range(40):
        assert q[n, int(np.argmin(w[:, n]))] == 0 and q[n, int(np.argmax(w[:, n]))] == 15
    deq = (q - zp[:, None].astype(np.int64)) / sa.astype(np.float64)[:, None]
    err = np.abs(w.T.astype(np.float64) - deq)
    step = 1.0 / sa.astype(np.float64)[:, None]
    assert (err <= step * (1 + 1e-6)).all()
    assert (err <= 0.5 * step * (1 + 1e-6)).mean() > 0.99


def test_w4z_scale_is_15_over_range_and_power_of_two_invariance():
    w = _random_w(k=200, n=8, seed=42)
    wp, sa, zp = oracle.w4z_quantize_pack(w)
    rng_ = (w.max(axis=0) - w.min(axis=0)).astype(np.float32)
    assert np.array_equal(sa, (np.float32(15.0) / rng_).astype(np.float32))
    for j in (-3, 2):
        wj, saj, zpj = oracle.w4z_quantize_pack((w * np.float32(2.0 ** j)).astype(np.float32))
        assert np.array_equal(wj, wp) and np.array_equal(zpj, zp)
        assert np.array_equal(saj * np.float32(2.0 ** j), sa)


def test_w4z_constant_and_positive_columns():
    """A constant column c has no range: sa = 1, zp = -rne(c), all codes 0,
    dequantized rne(c). An all-positive column gets a negative zero point and
    still spans codes 0..15."""
    w = np.zeros((6, 2), np.float32)
    w[:, 0] = 3.25
    w[:, 1] = [100.0, 100.2, 100.4, 100.6, 100.8, 101.0]
    wp, sa, zp = oracle.w4z_quantize_pack(w)
    assert sa[0] == 1.0 and zp[0] == -3 and not (wp[0] & 0x0F).any() and not (wp[0] >> 4).any()
    q = _unpack_unsigned(wp, 6)
    assert zp[1] < 0 and q[1, 0] == 0 and q[1, 5] == 15


def test_gemm_z_matches_float64_matmul():
    """sum_k xq * (q - zp) against float64 matmul of independently unpacked
    codes (exact while |acc| < 2^53)."""
    rng = synth.rng_for(43, 0)
    for (m, k, n) in ((1, 1, 1), (3, 7, 5), (24, 777, 40)):
        w = rng.normal(0.0, 0.02, size=(k, n)).astype(np.float32)
        wp, sa, zp = oracle.w4z_quantize_pack(w)
        xq = rng.integers(-127, 128, size=(m, k)).astype(np.int8)
        acc = oracle.gemm_z_s32(xq, k, wp, zp)
        q = _unpack_unsigned(wp, k) - zp[:, None].astype(np.int64)
        assert np.array_equal(acc.astype(np.float64), xq.astype(np.float64) @ q.T.astype(np.float64))


def test_linear_z_error_bound_and_tighter_than_symmetric():
    """|y - X @ W| within the bound with e_w = 1 / sa (the clamp case) and
    e_x = 0.5 / sx; and since the asymmetric grid spends all 16 levels on each
    column's range, its mean error on the same data is below the symmetric
    layer's (which uses 15 of 16 levels over twice the abs-max)."""
    x, _ = synth.linear_activations(8, 640, seed=44, outlier_count=3, outlier_factor=20.0)
    w = synth.linear_weights(640, 48, 0.02, seed=44)
    wp, sa, zp = oracle.w4z_quantize_pack(w)
    xq, sx = oracle.a8_quantize_rows(x)
    y = oracle.linear_z(x, wp, sa, zp, 640)
    x64, w64 = x.astype(np.float64), w.astype(np.float64)
    exact = x64 @ w64
    ew = 1.0 / sa.astype(np.float64)
    ex = 0.5 / sx.astype(np.float64)
    bound = (np.abs(x64).sum(1)[:, None] * ew[None, :] + ex[:, None] * np.abs(w64).sum(0)[None, :]
             + 640 * ex[:, None] * ew[None, :])
    slack = 1e-5 * (np.abs(x64) @ np.abs(w64)) + 1e-6
    assert (np.abs(y - exact) <= bound + slack).all()
    wps, sws = oracle.w4_quantize_pack(w)
    ys = oracle.linear(x, wps, sws, 640)
    assert np.abs(y - exact).mean() < np.abs(ys - exact).mean()


# ---------------------------------------------------- group-wise INT4 ---
# "INT4" concept page, section 4.2 (group quantization: each group of
# group_size weights has its own scale and zero point).

def test_w4g_hand_worked_two_groups():
    """K = 6, G = 4: group 0 = [-1, 0, 2, 0.5] -> sa 5, zp 5, codes 0 5 15 7;
    group 1 = [10, 20] (ragged) -> sa 15/10 = 1.5, zp -rne(15) = -15, codes 0, 15.
    With X = ones (sx = 127, codes 127) the partial sums are 127 * 7 = 889 and
    127 * 45 = 5715, and y = fl(fl(889 / 635) + fl(5715 / 190.5))."""
    w = np.array([[-1.0], [0.0], [2.0], [0.5], [10.0], [20.0]], np.float32)
    wp, sa, zp = oracle.w4g_quantize_pack(w, 4)
    assert sa.tolist() == [[5.0, 1.5]] and zp.tolist() == [[5, -15]]
    assert wp[0, :3].tolist() == [80, 127, 240] and not wp[0, 3:].any()
    y, acc = oracle.linear_g(np.ones((1, 6), np.float32), wp, sa, zp, 6, 4, partials=True)
    assert acc.tolist() == [[[889, 5715]]]
    f = np.float32
    assert y[0, 0] == f(f(f(889) / f(635)) + f(f(5715) / f(190.5)))


def test_w4g_one_group_is_the_per_channel_zero_point_layer():
    """G >= K leaves one group per channel: codes, scales, zero points,
    accumulators and outputs are those of the per-channel zero-point layer."""
    x, _ = synth.linear_activations(5, 300, seed=51, outlier_count=3, outlier_factor=20.0)
    w = synth.linear_weights(300, 24, 0.02, seed=51)
    b = synth.bias_vector(24, 51)
    wpz, saz, zpz = oracle.w4z_quantize_pack(w)
    for g in (300, 512):
        wp, sa, zp = oracle.w4g_quantize_pack(w, g)
        assert np.array_equal(wp, wpz) and np.array_equal(sa[:, 0], saz) and np.array_equal(zp[:, 0], zpz)
        y, acc = oracle.linear_g(x, wp, sa, zp, 300, g, bias=b, relu=True, partials=True)
        assert np.array_equal(acc[:, :, 0], oracle.linear_z(x, wpz, saz, zpz, 300, out="s32"))
        assert np.array_equal(y, oracle.linear_z(x, wpz, saz, zpz, 300, bias=b, relu=True))


def test_w4g_groups_are_independent_and_dequantize_within_a_step():
    """Changing the weights of one group changes no other group's codes or
    scales; every weight dequantizes within 1 / sa of its group."""
    k, n, G = 640, 16, 128
    w = _random_w(k=k, n=n, seed=52)
    wp, sa, zp = oracle.w4g_quantize_pack(w, G)
    w2 = w.copy()
    w2[256:384] *= np.float32(3.0)  # group 2 only
    wp2, sa2, zp2 = oracle.w4g_quantize_pack(w2, G)
    q = _unpack_unsigned(wp, k)
    q2 = _unpack_unsigned(wp2, k)
    others = np.r_[0:256, 384:640]
    assert np.array_equal(q[:, others], q2[:, others])
    assert np.array_equal(np.delete(sa, 2, axis=1), np.delete(sa2, 2, axis=1))
    assert np.array_equal(np.delete(zp, 2, axis=1), np.delete(zp2, 2, axis=1))
    g_of_k = np.arange(k) // G
    deq = (q - zp[:, g_of_k].astype(np.int64)) / sa[:, g_of_k].astype(np.float64)
    assert (np.abs(w.T.astype(np.float64) - deq) <= (1.0 / sa[:, g_of_k].astype(np.float64)) * (1 + 1e-6)).all()


def test_w4g_output_is_the_float32_sum_of_group_terms():
    """y against the float64 sum of the same per-group terms (from the INT32
    partials): float32 rounding of ng quotients and ng additions stays within
    (2 ng + 2) * 2^-24 of the sum of |terms|; and the partials sum to an exact
    float64 matmul of the dequantization-free integer form."""
    k, n, G = 1000, 20, 128
    x, _ = synth.linear_activations(6, k, seed=53, outlier_count=4, outlier_factor=20.0)
    w = synth.linear_weights(k, n, 0.02, seed=53)
    wp, sa, zp = oracle.w4g_quantize_pack(w, G)
    y, acc = oracle.linear_g(x, wp, sa, zp, k, G, partials=True)
    xq, sx = oracle.a8_quantize_rows(x)
    ng = sa.shape[1]
    terms = acc.astype(np.float64) / (sx.astype(np.float64)[:, None, None] * sa.astype(np.float64)[None, :, :])
    ref = terms.sum(axis=2)
    tol = (2 * ng + 2) * 2.0 ** -24 * np.abs(terms).sum(axis=2)
    assert (np.abs(y - ref) <= tol).all()
    q = _unpack_unsigned(wp, k) - zp[:, np.arange(k) // G].astype(np.int64)
    for g in range(ng):
        ks = slice(g * G, min(k, (g + 1) * G))
        assert np.array_equal(acc[:, :, g].astype(np.float64),
                              xq[:, ks].astype(np.float64) @ q[:, ks].T.astype(np.float64))


def test_w4g_error_below_per_channel_zero_point():
    """Finer groups, finer grids: on the same data the group-wise layer's mean
    error against X @ W is below the per-channel zero-point layer's."""
    x, _ = synth.linear_activations(8, 1024, seed=54, outlier_count=3, outlier_factor=20.0)
    w = synth.linear_weights(1024, 48, 0.02, seed=54)
    exact = x.astype(np.float64) @ w.astype(np.float64)
    wp, sa, zp = oracle.w4g_quantize_pack(w, 128)
    yg = oracle.linear_g(x, wp, sa, zp, 1024, 128)
    wpz, saz, zpz = oracle.w4z_quantize_pack(w)
    yz = oracle.linear_z(x, wpz, saz, zpz, 1024)
    assert np.abs(yg - exact).mean() < np.abs(yz - exact).mean()


def test_zero_point_storage_identity():
    """The algebra the zero-point kernels rely on, on the oracle alone: storing
    each code as the signed nibble q - 8 and multiplying with the symmetric
    INT4 product gives acc' = sum xq (q - 8); adding -(zp - 8) * sum xq gives
    sum xq (q - zp), the zero-point product, exactly."""
    rng = synth.rng_for(60, 0)
    k, n, m = 333, 24, 7
    w = rng.normal(0.0, 0.02, size=(k, n)).astype(np.float32)
    w[:, 3] = np.abs(w[:, 3]) + 1.0  # a negative zero point
    wp, sa, zp = oracle.w4z_quantize_pack(w)
    q = _unpack_unsigned(wp, k)
    stored = oracle.w4_pack((q - 8).astype(np.int8))  # signed nibbles q - 8, pad 0
    xq = rng.integers(-127, 128, size=(m, k)).astype(np.int8)
    acc_prime = oracle.gemm_s32(xq, k, stored).astype(np.int64)
    rowsum = xq.astype(np.int64).sum(axis=1)
    acc = acc_prime - (zp.astype(np.int64)[None, :] - 8) * rowsum[:, None]
    assert np.array_equal(acc, oracle.gemm_z_s32(xq, k, wp, zp).astype(np.int64))
