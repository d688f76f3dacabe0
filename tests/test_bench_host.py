"""Host-side pieces of bench.py: the max-over-ranks timing reduction on two
gloo ranks, and the CPU-oracle reference line."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from tests.conftest import ROOT

sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        got = bench.max_over_ranks(torch, dist, 10.0 + rank * 5.0, torch.device("cpu"))
        q.put((rank, got))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo_two_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert res == {0: 15.0, 1: 15.0}


def test_max_over_ranks_single_process_is_identity():
    assert bench.max_over_ranks(torch, None, 3.5, None) == 3.5


def test_reference_arm_prints_one_json_line():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--steps", "10", "--warmup", "3", "--cpu-budget", "0.5"],
                         capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert out.returncode == 0, out.stderr
    lines = [l for l in out.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "impl", "cpu_baseline", "e2e"):
        assert key in d
    assert d["impl"] == "reference" and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0


def test_reference_arm_other_ranks_exit_quietly():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--steps", "10", "--warmup", "3", "--cpu-budget", "0.5"],
                         capture_output=True, text=True, timeout=120, cwd=ROOT, env=env)
    assert out.returncode == 0 and out.stdout.strip() == ""


class _FakeLib:
    @staticmethod
    def w4z_workspace_size(m, k, n):
        return 64


class _FakeNative:
    """Stands in for the library on CPU: right shapes and dtypes, no arithmetic."""
    lib = _FakeLib()

    @staticmethod
    def packed_ld(k):
        return ((k + 1) // 2 + 15) // 16 * 16

    @staticmethod
    def w8a8_ld(k):
        return (k + 15) // 16 * 16

    @staticmethod
    def workspace_size(m, k):
        return 64

    def w4_quantize_pack(self, w):
        k, n = w.shape
        return torch.zeros((n, self.packed_ld(k)), dtype=torch.uint8), torch.ones(n)

    def w8_quantize(self, w):
        k, n = w.shape
        return torch.zeros((n, self.w8a8_ld(k)), dtype=torch.int8), torch.ones(n)

    def w4z_quantize_pack(self, w):
        k, n = w.shape
        return torch.zeros((n, self.packed_ld(k)), dtype=torch.uint8), torch.ones(n), torch.zeros(n, dtype=torch.int32)

    def w4g_quantize_pack(self, w):
        k, n = w.shape
        ng = -(-k // 128)
        return (torch.zeros((n, self.packed_ld(k)), dtype=torch.uint8), torch.ones((n, ng)),
                torch.zeros((n, ng), dtype=torch.int32))


@pytest.mark.parametrize("form", ["w4", "w8", "zp", "grp"])
def test_decode_workload_counts_the_bytes_each_form_moves(form):
    """The decode line's GB/s divide these bytes: per call the weights (packed
    INT4 rows, or INT8 rows), their scales (and zero points, per channel or
    per group of 128), the float32 activations and the float32 outputs."""
    from w4a8_quantized_gemm_channel_b200 import synth
    wl = bench.DecodeWorkload(torch, _FakeNative(), synth, torch.device("cpu"), 1 << 20,
                              w8=form == "w8", zp=form == "zp", grp=form == "grp")
    k, n = synth.DECODE_K, synth.DECODE_N
    ld = (k + 15) // 16 * 16 if form == "w8" else ((k + 1) // 2 + 15) // 16 * 16
    scales = {"w4": 4 * n, "w8": 4 * n, "zp": 8 * n, "grp": 8 * n * (-(-k // 128))}[form]
    want = sum(n * ld + scales + 4 * m * k + 4 * m * n for m in synth.DECODE_MS)
    assert wl.bytes_per_step() == want
    # the rotating weight copies exceed three times the L2 size, so every launch streams from HBM
    assert wl.pool_bytes >= 3 * (1 << 20) and len(wl.wp) == wl.pool
