"""The bench's roofline arithmetic on CPU: the algorithmic bytes and flops per
launch behind every achieved figure, and the whole-step roofline."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from post_weight_quantization_philox_b200 import synth  # noqa: E402


class _Layer:
    def __init__(self, L):
        self.L = L


@pytest.mark.parametrize("name,L,per_coord", [
    # 4 dW + 2 W_hat + logits and momenta read and written (16 L), + 1 initial
    # level for the 3-bit grid: the algorithmic bytes 4 + 16 L (+1) of the
    # backward plus the 2 B of the fused next soft weight
    ("c2_qproj_4096x4096", 4, 70), ("c4_gateproj_14336x4096", 4, 70),
    ("c3_downproj_4096x14336", 5, 87)])
def test_fused_backward_bytes_per_coordinate(name, L, per_coord):
    cfg = synth.CONFIGS[name]
    w = bench.phase_bytes_flops(cfg, _Layer(L), 4)
    groups = cfg.N * cfg.K // 128
    assert w["backward_lion_next_soft"] == ("hbm", cfg.N * cfg.K * per_coord + 16 * groups)
    # without the next soft weight: no W_hat
    assert w["backward_lion"][1] == cfg.N * cfg.K * (per_coord - 2) + 16 * groups
    # the soft weight alone: logits read, bf16 weight written (4 L + 2, + 1)
    extra = 1 if L == 5 else 0
    assert w["soft_weight"][1] == cfg.N * cfg.K * (4 * L + 2 + extra) + 4 * groups
    assert w["forward_gemm"] == ("tensor", 2.0 * cfg.N * cfg.T * cfg.K)
    assert w["weight_grad_gemm"] == w["forward_gemm"]


def test_bf16_state_halves_the_state_bytes():
    cfg = synth.CONFIGS["c2_qproj_4096x4096"]
    w32 = bench.phase_bytes_flops(cfg, _Layer(4), 4)["backward_lion_next_soft"][1]
    w16 = bench.phase_bytes_flops(cfg, _Layer(4), 2)["backward_lion_next_soft"][1]
    # logits and momenta, read and written: 4 planes x 4 logits x 2 bytes saved
    assert w32 - w16 == cfg.N * cfg.K * 32


def test_step_roofline_q_proj():
    cfg = synth.CONFIGS["c2_qproj_4096x4096"]
    w = bench.phase_bytes_flops(cfg, _Layer(4), 4)
    r = bench.step_roofline(w, 0.5, 1662.4, 6457.4)
    gemm_ms = 2 * 2 * 4096 ** 3 / 1662.4e12 * 1e3
    hbm_ms = w["backward_lion_next_soft"][1] / 6457.4e9 * 1e3
    assert r["gemm_ms"] == pytest.approx(gemm_ms, abs=1e-4)
    assert r["hbm_ms"] == pytest.approx(hbm_ms, abs=1e-4)
    assert r["frac"] == pytest.approx((gemm_ms + hbm_ms) / 0.5, abs=1e-4)
    # the whole-job rate counts every rank's units over the slowest rank's time
    assert bench.whole_job_rate(4, 10.0, 2.0) == pytest.approx(4 * 10.0 / 2e-3)


def test_block_step_accounting():
    """The 70B block step: seven weights, 8.55e8 coordinates per step; the
    fused backward's algorithmic bytes are 70 B per coordinate (2-bit, with
    the next soft weight) plus 16 B per group; the GEMM flops per stage."""
    dm = bench.BLOCK_70B
    dims = (dm["nseq"], dm["S"], dm["nh"], dm["nkv"], dm["d"], dm["F"])
    c = bench.block_step_coords(*dims)
    assert c == [8192 * 8192, 1024 * 8192, 1024 * 8192 + 8192 * 8192, 3 * 8192 * 28672]
    assert sum(c) == 855638016
    assert bench.block_backward_bytes(128) == 128 * 70 + 16
    assert bench.block_backward_bytes(128, next_soft=False) == 128 * 68 + 16
    f = bench.block_step_flops(*dims)
    T = 8 * 2048
    assert f[0] == 4.0 * T * 8192 * 8192 and f[1] == 4.0 * T * 1024 * 8192
    assert f[3] == 14.0 * T * 8192 * 28672


def test_traffic_counters_follow_the_code_not_the_comments():
    a = "int f(int x) {  // doubles\n  return 2 * x; /* fast */ }\n"
    b = "int f(int x) {  // twice x\n\n  return 2 * x;   }\n"
    c = "int f(int x) {  // doubles\n  return 3 * x; /* fast */ }\n"
    assert bench.code_hash([a]) == bench.code_hash([b])
    assert bench.code_hash([a]) != bench.code_hash([c])
