"""w4a8_linear_noalloc: the entry point for callers that cannot allocate
device memory (for example a host that passes the library only its input and
output buffers). It keeps the INT8 activations in a fixed scratch array the
library owns instead of a caller workspace, and must give the same results as
w4a8_linear. This file is collected last on purpose, so a run that stops at
the first failure has already run every other test.
"""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

RTOL = 1e-6


def _close(y, ref):
    y = np.asarray(y, np.float64)
    ref = np.asarray(ref, np.float64)
    assert (np.abs(y - ref) <= RTOL * np.abs(ref)).all()


def test_noalloc_matches_linear_on_two_calls_in_a_row():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from w4a8_quantized_gemm_channel_b200 import native, synth

    native.get_device_status(clear=True)
    cases = []
    # a decode-shaped call, then a smaller tensor-core call: the second must
    # not see anything the first left in the shared scratch array
    for (m, k, n, seed) in ((16, 4096, 1024, 31), (300, 520, 300, 32)):
        w = synth.linear_weights(k, n, 0.02, seed)
        x, _ = synth.linear_activations(m, k, seed, outlier_count=4, outlier_factor=20.0)
        b = synth.bias_vector(n, seed)
        wp, sw = native.w4_quantize_pack(torch.from_numpy(w).cuda())
        xd, bd = torch.from_numpy(x).cuda(), torch.from_numpy(b).cuda()
        cases.append((xd, wp, sw, bd))
    for xd, wp, sw, bd in cases:
        got = native.w4a8_linear_noalloc(xd, wp, sw, bias=bd, relu=True)
        want = native.w4a8_linear(xd, wp, sw, bias=bd, relu=True)
        torch.cuda.synchronize()
        _close(got.cpu().numpy(), want.cpu().numpy())
        acc = native.w4a8_linear_noalloc(xd, wp, sw, out="s32")
        acc_want = native.w4a8_linear(xd, wp, sw, out="s32")
        torch.cuda.synchronize()
        assert torch.equal(acc, acc_want)
    assert native.get_device_status() == 0


def test_noalloc_rejects_sizes_beyond_the_scratch_array():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from w4a8_quantized_gemm_channel_b200 import native

    k = 4096
    m = native.NOALLOC_SCRATCH_BYTES // k + 1      # needs more than the array holds
    assert native.workspace_size(m, k) > native.NOALLOC_SCRATCH_BYTES
    x = torch.zeros((m, k), device="cuda")
    wp = torch.zeros((8, native.packed_ld(k)), dtype=torch.uint8, device="cuda")
    sw = torch.ones(8, device="cuda")
    with pytest.raises(native.W4A8Error) as e:
        native.w4a8_linear_noalloc(x, wp, sw)
    assert e.value.status == native.ERR_WORKSPACE
